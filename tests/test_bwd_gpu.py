"""GPU parity of attn_bwd (prep, backward and dQ conversion kernels, through
the C ABI) against the fp64 oracle's gradients (oracle.attention_bwd).

Tolerances, per gradient tensor, against the unrounded fp64 oracle:
  ||g - g*||_2 / ||g*||_2 <= 5e-3   and   max |g - g*| <= 2^-6 * max |g*|
Derivation: the kernels round P to bf16 before dV = P^T dO and inside
dS = P (dP - Drow), round dS to bf16 before dK and dQ, and round each output
to bf16 once; every other step accumulates in fp32.  Each rounding has
relative error at most 2^-8 (RMS about 1.1e-3), so dQ and dK carry three of
them (RMS about 1.9e-3 relative), dV two; 5e-3 leaves more than 2.5x margin.
The largest element's own output rounding is at most 2^-8 of it; 2^-6 bounds
it with the arithmetic before it.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import to_np64

pytestmark = pytest.mark.gpu

G_REL_RMS = 5e-3
G_MAX_ABS_FRAC = 2.0 ** -6
ZERO_GRAD_ABS = 1e-4


def _grads_check(got, ref, what):
    g = to_np64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    scale = float(np.abs(ref).max())
    err = float(np.abs(g - ref).max())
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / nrm) if nrm > 0 else float(np.linalg.norm(g))
    print(f"{what}: max_abs={err:.3e} (max|ref|={scale:.3e}) rel_rms={rel:.3e}")
    if nrm == 0:
        # The exact gradient is 0 (e.g. one key: dS = P (dP - Drow) with P = 1
        # and dP = Drow).  The kernel forms dP on the tensor core and Drow with
        # FMAs from the same bf16 values, so the two differ by fp32 rounding
        # (~D * 2^-24 * sum |dO V|), which dQ = scale * dS K carries on.
        assert err <= ZERO_GRAD_ABS, f"{what}: {err:.3e} where the exact gradient is 0"
        return
    assert rel <= G_REL_RMS, f"{what}: rel_rms {rel:.3e} > {G_REL_RMS}"
    assert err <= G_MAX_ABS_FRAC * scale, f"{what}: max_abs {err:.3e} > {G_MAX_ABS_FRAC} * {scale:.3e}"


def _run(q, k, v, do, causal, scale):
    d = torch.device("cuda:0")
    q, k, v, do = (t.to(d) for t in (q, k, v, do))
    o, lse = ea.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = ea.bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    return dq, dk, dv


def _check(B, Hq, Hkv, Nq, Nk, D, causal, seed):
    q, k, v, do = inputs.bwd_inputs(B, Hq, Hkv, Nq, Nk, D, seed)
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = _run(q, k, v, do, causal, scale)
    rq, rk, rv = oracle.attention_bwd(to_np64(q), to_np64(k), to_np64(v), to_np64(do), causal, scale)
    tag = f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} D{D} causal={causal}"
    _grads_check(dq, rq, "dQ " + tag)
    _grads_check(dk, rk, "dK " + tag)
    _grads_check(dv, rv, "dV " + tag)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_square_multi_block(D, causal):
    _check(2, 2, 2, 384, 384, D, causal, seed=D + causal)


@pytest.mark.parametrize("D", [64, 128])
def test_gqa_ragged(D):
    """Four query heads per KV head; neither length a multiple of the block."""
    _check(1, 8, 2, 300, 300, D, True, seed=7 + D)


@pytest.mark.parametrize("Nq,Nk,causal", [(200, 333, True), (333, 200, False), (300, 130, True), (1, 257, True),
                                          (257, 1, False), (129, 129, True)])
def test_unequal_lengths(Nq, Nk, causal):
    """Bottom-right causal alignment; with Nq > Nk the first rows see no key."""
    _check(1, 4, 1, Nq, Nk, 128, causal, seed=Nq * 3 + Nk)


@pytest.mark.parametrize("D,Nq", [(64, 2048), (128, 2000)])
def test_many_query_blocks_per_key_block(D, Nq):
    """A long non-causal case: each CTA walks 16 (D = 64) or 32 (D = 128)
    query blocks x 2 heads; 2000 queries leave a ragged last block and a
    padded accumulator row."""
    _check(1, 4, 2, Nq, 256, D, False, seed=31 + D)


@pytest.mark.parametrize("D", [64, 128])
def test_empty_query_or_key_side(D):
    d = torch.device("cuda:0")
    q, k, v, do = inputs.bwd_inputs(1, 2, 1, 0, 130, D, 3)
    q, k, v, do = (t.to(d) for t in (q, k, v, do))
    o = torch.empty_like(q)
    lse = torch.empty(1, 2, 0, device=d)
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(v, 7.0)
    ea.bwd(q, k, v, o, lse, do, causal=True, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    assert not dk.any() and not dv.any()          # no query: zero gradients for K and V
    q, k, v, do = inputs.bwd_inputs(1, 2, 1, 70, 0, D, 4)
    q, k, v, do = (t.to(d) for t in (q, k, v, do))
    o, lse = ea.fwd(q, k, v, causal=False)
    dq = torch.full_like(q, 7.0)
    ea.bwd(q, k, v, o, lse, do, dq=dq)
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    assert not dq.any()                           # no key: zero gradient for Q


def test_dk_dv_deterministic():
    q, k, v, do = inputs.bwd_inputs(1, 4, 2, 500, 500, 128, 12)
    a = _run(q, k, v, do, True, 0.09)
    b = _run(q, k, v, do, True, 0.09)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_workspace_errors():
    d = torch.device("cuda:0")
    q, k, v, do = (t.to(d) for t in inputs.bwd_inputs(1, 2, 1, 130, 130, 64, 5))
    o, lse = ea.fwd(q, k, v)
    need = ea.bwd_workspace_size(1, 2, 130, 64)
    assert need >= 1 * 130 * 2 * 64 * 4
    ws = torch.empty(need, dtype=torch.uint8, device=d)
    lib = ea.library()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    args = [t.data_ptr() for t in (q, k, v, o, do, lse, dq, dk, dv)] + [1, 2, 1, 130, 130, 64, 64, 0, 0.125]
    stream = torch.cuda.current_stream(d).cuda_stream
    assert lib.attn_bwd(*args, ws.data_ptr(), need - 256, stream) == 5
    assert lib.attn_bwd(*args, None, need, stream) == 5
    assert lib.attn_bwd(*args, ws.data_ptr(), need, stream) == 0
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0


def test_long_context_gqa_workload_sampled():
    """The long-context GQA causal shape (B1, Hq32, Hkv8, N16384, D128) in the
    launch configuration the bench times: dQ of sampled query rows and dK, dV
    of sampled key rows of KV head 3 (its four query heads), against the
    oracle, which still uses every query row for those key rows."""
    cfg = inputs.PREFILL_CONFIGS[3]
    q, k, v, do = inputs.bwd_config_inputs(cfg)
    dq, dk, dv = _run(q, k, v, do, cfg.causal, cfg.scale)
    N = cfg.Nq
    rows = np.array([0, 1, 127, 128, 4095, 8191, 8192, 12000, N - 129, N - 2, N - 1])
    keys = np.array([0, 5, 127, 128, 2048, 8190, 12345, N - 200, N - 128, N - 1])
    rq, rk, rv = oracle.attention_bwd(to_np64(q), to_np64(k), to_np64(v), to_np64(do), cfg.causal, cfg.scale,
                                      q_rows=rows, k_rows=keys, kv_heads=[3])
    dq, dk, dv = (t.cpu() for t in (dq, dk, dv))
    r, kk = torch.as_tensor(rows), torch.as_tensor(keys)
    _grads_check(dq[:, r, 12:16], rq[:, :, 12:16], "dQ long-context sampled rows, heads 12-15")
    _grads_check(dk[:, kk, 3], rk[:, :, 3], "dK long-context sampled keys, KV head 3")
    _grads_check(dv[:, kk, 3], rv[:, :, 3], "dV long-context sampled keys, KV head 3")


@pytest.mark.parametrize("D", [64, 128])
def test_head_grouped_unit_order_sampled(D):
    """Non-causal, B1, Hq = Hkv = 3, N = 9600: 75 key blocks per head, so the
    unit order takes the heads two at a time (ceil(148 / 75) = 2, and with
    equal units grouping costs nothing), which leaves a last group of one
    head.  dQ of sampled query rows of every head, and dK, dV of sampled key
    rows of the last group's head (2) and of the first group's second head (1),
    against the oracle."""
    N, H = 9600, 3
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = inputs.bwd_inputs(1, H, H, N, N, D, seed=97)
    dq, dk, dv = _run(q, k, v, do, False, scale)
    rows = np.array([0, 1, 63, 64, 4800, N - 65, N - 1])
    keys = np.array([0, 127, 128, 5000, 9471, 9472, N - 1])
    for kvh in (2, 1):
        rq, rk, rv = oracle.attention_bwd(to_np64(q), to_np64(k), to_np64(v), to_np64(do), False, scale,
                                          q_rows=rows, k_rows=keys, kv_heads=[kvh])
        r, kk = torch.as_tensor(rows), torch.as_tensor(keys)
        _grads_check(dq.cpu()[:, r, kvh], rq[:, :, kvh], f"dQ sampled rows, head {kvh}, D={D}")
        _grads_check(dk.cpu()[:, kk, kvh], rk[:, :, kvh], f"dK sampled keys, KV head {kvh}, D={D}")
        _grads_check(dv.cpu()[:, kk, kvh], rv[:, :, kvh], f"dV sampled keys, KV head {kvh}, D={D}")
