"""GPU parity of attn_fwd_fp8 (through the C ABI) against the fp64 oracle on
the values the E4M3 inputs represent (oracle.attention_fp8).

Tolerances, derived from the kernel's own roundings (the inputs themselves
are exact: every e4m3 product is exact in fp32):
  * each probability is rounded to e4m3 before the product with V.  The
    kernel measures p from 2^4 below the row's reference max, so p lies in
    (0, 256] and all but negligible weights are e4m3 normals, with relative
    error at most 2^-4 (RMS about 2.6e-2 over uniformly spread mantissas).
    O therefore moves by at most 2^-4 * max|V| per element, plus its own bf16
    rounding (2^-8 * |O|): max-abs <= (2^-4 + 2^-8) * max|V|.  With weights
    and V rows independent, the relative RMS of O's error equals the RMS of
    the weights' relative errors: rel-RMS <= 5e-2 (about 2x margin).
  * the row sums and the LSE use the unrounded fp32 probabilities: LSE
    max-abs <= 1e-3 as in the bf16 path.
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

O_REL_RMS = 5e-2
P_ROUND = 2.0 ** -4 + 2.0 ** -8
LSE_MAX_ABS = 1e-3


def _run(q8, k8, v8, ds, causal, scale):
    dev = torch.device("cuda:0")
    o, lse = ea.fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *ds, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    return o, lse


def _compare(o, lse, o_ref, lse_ref, vmax, what):
    o = to_np64(o)
    lse = to_np64(lse)
    assert np.all(np.isfinite(o)), what
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref)), what
    fin = np.isfinite(lse_ref)
    lse_err = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    err = float(np.abs(o - o_ref).max())
    nrm = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref) / nrm) if nrm > 0 else 0.0
    print(f"{what}: max_abs={err:.3e} (bound {P_ROUND * vmax:.3e}) rel_rms={rel:.3e} lse={lse_err:.2e}")
    assert err <= P_ROUND * vmax, what
    assert rel <= O_REL_RMS, what
    assert lse_err <= LSE_MAX_ABS, what


def _check(B, Hq, Hkv, Nq, Nk, causal, seed):
    q8, k8, v8, ds = inputs.fp8_prefill_inputs(B, Hq, Hkv, Nq, Nk, 128, seed)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run(q8, k8, v8, ds, causal, scale)
    o_ref, lse_ref = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), *ds, causal, scale)
    vmax = ds[2] * float(np.nanmax(np.abs(oracle.e4m3_decode(v8.numpy())))) if Nk else 0.0
    _compare(o, lse, o_ref, lse_ref, vmax, f"fp8 B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} causal{causal}")


SHAPES = [
    # B, Hq, Hkv, Nq, Nk, causal
    (1, 2, 2, 128, 128, False),
    (2, 4, 2, 200, 333, False),
    (2, 4, 2, 200, 333, True),        # Nq < Nk, bottom-right causal
    (1, 2, 1, 300, 130, True),        # Nq > Nk: leading rows see no key
    (1, 4, 4, 640, 640, True),
    (1, 8, 8, 1, 1000, False),        # one query row
    (1, 1, 1, 130, 1, False),         # one key
    (1, 4, 1, 1029, 1029, True),      # many key blocks, ragged
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_Hq{}_Hkv{}_Nq{}_Nk{}_c{}".format(*s))
def test_shapes(shape):
    _check(*shape, seed=sum(shape[:5]) + 17)


def test_long_context_gqa_workload_sampled():
    """The long-context GQA causal shape (B1, Hq32, Hkv8, N16384, D128) in E4M3,
    in the launch configuration the bench times; sampled query rows of every
    head against the oracle."""
    cfg = inputs.PREFILL_CONFIGS[3]
    q8, k8, v8, ds = inputs.fp8_prefill_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.seed)
    o, lse = _run(q8, k8, v8, ds, cfg.causal, cfg.scale)
    rng = np.random.default_rng(cfg.seed)
    rows = np.array(sorted(set(rng.choice(cfg.Nq, 20, replace=False).tolist()) | {0, 1, 127, 128, cfg.Nq - 1}))
    o_ref, lse_ref = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), *ds, cfg.causal, cfg.scale,
                                          q_rows=rows)
    vmax = ds[2] * float(np.nanmax(np.abs(oracle.e4m3_decode(v8.numpy()))))
    r = torch.as_tensor(rows)
    _compare(o.cpu()[:, r], lse.cpu()[:, :, r], o_ref, lse_ref, vmax, "fp8 long-context GQA (sampled rows)")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_deterministic():
    q8, k8, v8, ds = inputs.fp8_prefill_inputs(1, 4, 2, 700, 700, 128, 23)
    o1, l1 = _run(q8, k8, v8, ds, True, 0.088)
    o2, l2 = _run(q8, k8, v8, ds, True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_unsupported_head_dim_is_rejected():
    dev = torch.device("cuda:0")
    q8, k8, v8, ds = inputs.fp8_prefill_inputs(1, 2, 1, 64, 64, 64, 2)
    with pytest.raises(ea.AttnError) as e:
        ea.fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *ds)
    assert e.value.code == 2
