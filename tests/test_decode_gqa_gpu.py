"""GPU parity of attn_decode_paged_gqa (decode kernel + LSE combine, through the
C ABI) against the fp64 oracle (oracle.decode_paged_gqa)."""

import math

import numpy as np
import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import bf16_arith_bound, compare, to_np64

pytestmark = pytest.mark.gpu

PAGE = 64


def _dev(c):
    d = torch.device("cuda:0")
    return (c.q.to(d), c.k_pages.to(d), c.v_pages.to(d), c.block_table.to(d), c.cache_seqlens.to(d))


def _run(c, scale):
    q, kp, vp, bt, sl = _dev(c)
    o, lse = ea.decode_paged_gqa(q, kp, vp, bt, sl, scale)
    torch.cuda.synchronize()
    return o, lse


def _oracle(c, scale, seqs=None):
    return oracle.decode_paged_gqa(to_np64(c.q)[:, 0], to_np64(c.k_pages), to_np64(c.v_pages), c.block_table.numpy(),
                                   c.cache_seqlens.numpy(), scale, page_size=PAGE, seqs=seqs)


def _vmax(c):
    """max |V| over rows that belong to a sequence (the sentinel rows carry weight 0)."""
    m = 0.0
    for b, L in enumerate(c.cache_seqlens.tolist()):
        t = torch.arange(L)
        if L:
            m = max(m, float(c.v_pages[c.block_table[b, t // PAGE].long(), t % PAGE].abs().max()))
    return m


def _check(lens, Hq, Hkv, D, seed, short=False):
    c = inputs.paged_gqa_decode_inputs(len(lens), Hq, Hkv, D, lens, PAGE, seed)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run(c, scale)
    assert ea.read_device_status(0) == 0
    o_ref, lse_ref = _oracle(c, scale)
    tol = dict(o_max_abs=bf16_arith_bound(_vmax(c))) if short else {}
    compare(o[:, 0], lse, o_ref, lse_ref, f"gqa decode Hq{Hq} Hkv{Hkv} D{D} lens={lens[:6]}", **tol)
    return c, o, lse


@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (8, 8, 128), (16, 8, 64), (16, 2, 128), (8, 4, 64), (4, 1, 128)])
def test_shapes(Hq, Hkv, D):
    # ragged last pages, an empty sequence, one page exactly, many pages
    _check([65, 0, 64, 1300, 7], Hq, Hkv, D, seed=Hq * 7 + Hkv + D, short=True)


@pytest.mark.parametrize("lens", [[1], [64], [8192], [3000, 17, 0, 4096, 64 * 37], [0, 0, 5]])
def test_lengths(lens):
    _check(lens, 32, 8, 128, seed=sum(lens) + 3, short=True)


def test_many_short_sequences():
    """Hundreds of short sequences: many units per worker, most written directly."""
    rng = np.random.default_rng(9)
    lens = rng.integers(0, 300, size=400).tolist()
    _check(lens, 32, 8, 128, seed=91, short=True)


def test_one_long_sequence_split_over_every_worker():
    """One sequence with one KV head: its single unit is cut into a piece per
    worker, so the combine kernel merges hundreds of partial results."""
    _check([64 * 600 + 5], 4, 1, 128, seed=5, short=False)


def test_gqa_workload_sampled_sequences():
    """The full GQA-path workload (B64, Hq32/Hkv8, D128, L ~ U[1024, 8192]),
    in the launch configuration the bench times; eight sequences, all heads,
    checked against the oracle."""
    cfg = inputs.GQA_DECODE_CONFIG
    c = inputs.gqa_decode_config_inputs()
    o, lse = _run(c, cfg.scale)
    assert ea.read_device_status(0) == 0
    seqs = [0, 1, 17, 31, 32, 50, 62, 63]
    o_ref, lse_ref = _oracle(c, cfg.scale, seqs=seqs)
    compare(o[seqs, 0], lse[seqs], o_ref, lse_ref, "gqa decode workload (sampled sequences)")


def test_deterministic_and_placement_invariant():
    lens = [700, 3, 1500, 64, 0, 2049]
    c = inputs.paged_gqa_decode_inputs(len(lens), 32, 8, 128, lens, PAGE, 13)
    o1, l1 = _run(c, 0.09)
    o2, l2 = _run(c, 0.09)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # move every page to another physical slot: the result must not change at all
    g = torch.Generator().manual_seed(3)
    perm = torch.randperm(c.num_pages, generator=g)
    kp, vp = torch.empty_like(c.k_pages), torch.empty_like(c.v_pages)
    kp[perm] = c.k_pages
    vp[perm] = c.v_pages
    c2 = inputs.PagedKV(c.q, kp, vp, perm.to(torch.int32)[c.block_table.long()], c.cache_seqlens, PAGE)
    o3, l3 = _run(c2, 0.09)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_bad_block_table_entry_reports_invalid_arg():
    lens = [200, 90]
    c = inputs.paged_gqa_decode_inputs(len(lens), 8, 2, 128, lens, PAGE, 21)
    bt = c.block_table.clone()
    bt[1, 0] = c.num_pages + 5
    c2 = inputs.PagedKV(c.q, c.k_pages, c.v_pages, bt, c.cache_seqlens, PAGE)
    o, lse = _run(c2, 0.1)
    assert ea.read_device_status(0) == 1
    # the other sequence is still exact
    o_ref, lse_ref = _oracle(c, 0.1, seqs=[0])
    compare(o[[0], 0], lse[[0]], o_ref, lse_ref, "gqa decode sequence next to a bad one",
            o_max_abs=bf16_arith_bound(_vmax(c)))


def test_workspace_too_small_is_rejected():
    c = inputs.paged_gqa_decode_inputs(2, 8, 2, 128, [100, 10], PAGE, 2)
    q, kp, vp, bt, sl = _dev(c)
    need = ea.decode_gqa_workspace_size(2, 8, 2, 128)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    o = torch.empty(2, 1, 8, 128, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(2, 8, dtype=torch.float32, device=q.device)
    lib = ea.library()
    args = (q.data_ptr(), kp.data_ptr(), vp.data_ptr(), bt.data_ptr(), sl.data_ptr(), o.data_ptr(), lse.data_ptr(),
            2, 8, 2, 128, PAGE, c.num_pages, bt.shape[1], 0.1, ws.data_ptr())
    stream = torch.cuda.current_stream(q.device).cuda_stream
    assert lib.attn_decode_paged_gqa(*args, need - 256, stream) == 5
    assert lib.attn_decode_paged_gqa(*args[:-1], None, need, stream) == 5
    assert lib.attn_decode_paged_gqa(*args, need, stream) == 0
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0


def test_maximum_batch_of_sequences():
    """B = 2048 short sequences (0..70 tokens), groups of 8: the largest batch."""
    rng = np.random.default_rng(41)
    lens = rng.integers(0, 71, size=2048).tolist()
    c = inputs.paged_gqa_decode_inputs(len(lens), 8, 1, 128, lens, PAGE, 41)
    o, lse = _run(c, 0.0883883)
    assert ea.read_device_status(0) == 0
    seqs = [0, 3, 777, 1024, 2047, int(np.argmax(lens))]
    o_ref, lse_ref = oracle.decode_paged_gqa(to_np64(c.q)[:, 0], to_np64(c.k_pages), to_np64(c.v_pages),
                                             c.block_table.numpy(), c.cache_seqlens.numpy(), 0.0883883,
                                             page_size=PAGE, seqs=seqs)
    compare(o[seqs, 0], lse[seqs], o_ref, lse_ref, "gqa decode B=2048", o_max_abs=bf16_arith_bound(_vmax(c)))
    empty = torch.tensor(lens) == 0
    assert torch.isneginf(lse.cpu()[empty]).all() and torch.isfinite(lse.cpu()[~empty]).all()
