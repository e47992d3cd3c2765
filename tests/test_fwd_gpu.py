"""GPU parity of attn_fwd (through the C ABI) against the fp64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import bf16_arith_bound, compare, to_np64

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, scale):
    dev = torch.device("cuda:0")
    o, lse = ea.fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    return o, lse


def _check_full(B, Hq, Hkv, Nq, Nk, D, causal, seed, q_mult=1.0, scale=None):
    q, k, v = inputs.prefill_inputs(B, Hq, Hkv, Nq, Nk, D, D, seed, q_mult)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = _run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention(to_np64(q), to_np64(k), to_np64(v), causal, scale)
    return compare(o, lse, o_ref, lse_ref, f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nk{Nk} D{D} causal{causal}")


def test_config1_tiny():
    cfg = inputs.PREFILL_CONFIGS[1]
    _check_full(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.causal, cfg.seed, scale=cfg.scale)


def test_config2_gpt2_small_causal():
    cfg = inputs.PREFILL_CONFIGS[2]
    _check_full(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.causal, cfg.seed, scale=cfg.scale)


SHAPES = [
    # B, Hq, Hkv, Nq, Nk, D, causal
    (1, 2, 2, 128, 128, 64, True),
    (2, 4, 2, 200, 333, 64, False),
    (2, 4, 2, 200, 333, 64, True),        # Nq < Nk, bottom-right causal
    (1, 2, 1, 300, 130, 128, True),       # Nq > Nk: leading rows see no key
    (1, 4, 1, 513, 515, 128, False),
    (1, 4, 4, 640, 640, 128, True),
    (2, 3, 1, 257, 190, 256, False),
    (1, 2, 2, 257, 257, 256, True),
    (1, 8, 8, 1, 1000, 128, False),       # one query row
    (1, 8, 2, 5, 7, 64, True),
    (1, 1, 1, 130, 1, 256, False),        # one key
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_Hq{}_Hkv{}_Nq{}_Nk{}_D{}_c{}".format(*s))
def test_shapes(shape):
    B, Hq, Hkv, Nq, Nk, D, causal = shape
    _check_full(B, Hq, Hkv, Nq, Nk, D, causal, seed=7 + Nq + Nk + D)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_growing_row_max_rescales(D):
    """Keys ordered so each block holds larger scores than the last: the row
    max keeps growing, so the O rescale path runs on every block."""
    B, H, N = 1, 2, 1024
    q, k, v = inputs.prefill_inputs(B, H, H, N, N, D, D, seed=99)
    ramp = torch.linspace(0.2, 3.0, N).view(1, N, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, scale)
        o_ref, lse_ref = oracle.attention(to_np64(q), to_np64(k), to_np64(v), causal, scale)
        compare(o, lse, o_ref, lse_ref, f"ramp D{D} causal{causal}",
                o_max_abs=bf16_arith_bound(v.float().abs().max().item()))


@pytest.mark.parametrize("D", [64, 128])
def test_persistent_walk_with_keyless_tiles(D):
    """More units than SMs (each CTA walks several), causal with Nq > Nk so
    that the first units' tiles see no key at all (O = 0, LSE = -inf) while
    later units of the same CTA do full work: the barrier counts that carry
    across units (Q tile free, O read, last product) must stay in step."""
    _check_full(4, 64, 8, 700, 300, D, True, seed=71 + D)


def test_no_keys():
    dev = torch.device("cuda:0")
    q, k, v = inputs.prefill_inputs(1, 2, 2, 100, 0, 128, 128, seed=3)
    o, lse = ea.fwd(q.to(dev), k.to(dev), v.to(dev), causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0)
    assert torch.all(torch.isneginf(lse))


def test_closed_forms_on_gpu():
    """Causal row 0 returns V[0]; a constant V row returns that row."""
    dev = torch.device("cuda:0")
    q, k, v = inputs.prefill_inputs(2, 4, 2, 384, 384, 128, 128, seed=5)
    o, lse = ea.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    torch.cuda.synchronize()
    kv_of = torch.arange(4) // 2
    assert torch.equal(o[:, 0].cpu(), v[:, 0, kv_of])
    row = torch.randn(128).to(torch.bfloat16)
    vc = row.view(1, 1, 1, 128).expand(2, 384, 2, 128).contiguous()
    o2, _ = ea.fwd(q.to(dev), k.to(dev), vc.to(dev), causal=False)
    torch.cuda.synchronize()
    assert (o2.cpu().float() - row.float()).abs().max().item() <= 2 ** -7 * row.float().abs().max().item()


def test_deterministic_and_guard_bands():
    dev = torch.device("cuda:0")
    B, Hq, Hkv, N, D = 2, 4, 2, 700, 128
    q, k, v = [t.to(dev) for t in inputs.prefill_inputs(B, Hq, Hkv, N, N, D, D, seed=11)]
    n_o = B * N * Hq * D
    n_l = B * Hq * N
    pad = 4096
    o_buf = torch.full((n_o + 2 * pad,), 123.0, dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((n_l + 2 * pad,), -55.0, dtype=torch.float32, device=dev)
    o = o_buf[pad:pad + n_o].view(B, N, Hq, D)
    lse = l_buf[pad:pad + n_l].view(B, Hq, N)
    ea.fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    first = (o.clone(), lse.clone())
    for _ in range(3):
        ea.fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(first[0], o) and torch.equal(first[1], lse)
    assert torch.all(o_buf[:pad] == 123.0) and torch.all(o_buf[pad + n_o:] == 123.0)
    assert torch.all(l_buf[:pad] == -55.0) and torch.all(l_buf[pad + n_l:] == -55.0)


def _sampled_rows(Nq, n, seed, causal):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(Nq, size=n, replace=False).tolist())
    rows |= {0, 1, 127, 128, Nq - 1}
    return np.array(sorted(r for r in rows if 0 <= r < Nq))


@pytest.mark.parametrize("cfg_id", [3, 4])
def test_full_size_configs_sampled(cfg_id):
    """Full-size workloads in the bench's launch configuration; the oracle
    recomputes a sample of query rows in every head."""
    cfg = inputs.PREFILL_CONFIGS[cfg_id]
    q, k, v = inputs.prefill_config_inputs(cfg)
    o, lse = _run(q, k, v, cfg.causal, cfg.scale)
    rows = _sampled_rows(cfg.Nq, 24, cfg.seed, cfg.causal)
    o_ref, lse_ref = oracle.attention(to_np64(q), to_np64(k), to_np64(v), cfg.causal, cfg.scale, q_rows=rows)
    compare(o[:, rows], lse[:, :, rows], o_ref, lse_ref, cfg.name)
    # properties at every row: finite output, |O| bounded by max |V| of its KV head
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    vmax = v.float().abs().amax().item()
    assert o.float().abs().max().item() <= vmax * (1 + 2 ** -7)


def test_error_codes_do_not_launch():
    dev = torch.device("cuda:0")
    q, k, v = [t.to(dev) for t in inputs.prefill_inputs(1, 3, 2, 64, 64, 64, 64, seed=1)]
    with pytest.raises(ValueError):
        ea.fwd(q, k[:, :, :1].contiguous(), v, causal=False)   # shape mismatch caught by the binding
    lib = ea.library()
    o = torch.full((1, 64, 3, 64), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 3, 64), dtype=torch.float32, device=dev)
    rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 3, 2, 64, 64, 64,
                      64, 0, 0.125, None)
    assert rc == 1   # Hq % Hkv != 0
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)
