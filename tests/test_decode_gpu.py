"""GPU parity of attn_decode_paged (split kernel + LSE combine, through the C ABI)
against the fp64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import bf16_arith_bound, compare, to_np64

pytestmark = pytest.mark.gpu

HQ, DK, DV, PAGE = 128, 576, 512, 64
SCALE = 1.0 / math.sqrt(192.0)


def _dev(c):
    d = torch.device("cuda:0")
    return (c.q.to(d), c.kv_pages.to(d), c.block_table.to(d), c.cache_seqlens.to(d))


def _run(c, scale=SCALE):
    q, kv, bt, sl = _dev(c)
    o, lse = ea.decode_paged(q, kv, bt, sl, scale, dv=DV)
    torch.cuda.synchronize()
    return o, lse


def _oracle(c, seqs=None, heads=None, scale=SCALE):
    seqs = list(range(c.q.shape[0])) if seqs is None else list(seqs)
    q = to_np64(c.q)[seqs, 0]
    pages = to_np64(c.kv_pages)[:, :, 0]
    return oracle.decode_paged(q, pages, c.block_table.numpy()[seqs], c.cache_seqlens.numpy()[seqs], scale, DV,
                               page_size=PAGE, heads=heads)


def _check(lens, seed, seqs=None, heads=None):
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    seqs = list(range(len(lens))) if seqs is None else list(seqs)
    o_ref, lse_ref = _oracle(c, seqs, heads)
    o_g = o[seqs, 0]
    l_g = lse[seqs]
    if heads is not None:
        o_g = o_g[:, heads]
        l_g = l_g[:, heads]
    return compare(o_g, l_g, o_ref, lse_ref, f"decode lens={lens[:6]}..."), c, o, lse


@pytest.mark.parametrize("lens", [
    [1],
    [64],
    [65, 1, 64, 127],
    [0, 100, 5000],
    [8192],                     # one long sequence: every CTA pair holds a piece of it
    [3000, 17, 0, 4096, 64 * 37],
])
def test_small_batches(lens):
    _check(lens, seed=sum(lens) + len(lens))


def test_many_short_sequences():
    """Hundreds of sequences of 0..199 tokens: many segments per CTA pair.
    Short rows give peaked softmax weights, so O is held to the bound of the
    kernel's own bf16 roundings (the workload tolerance is for the decode
    workload's lengths of 1024..8192)."""
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 200, size=300).tolist()
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=77)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    o_ref, lse_ref = _oracle(c)
    compare(o[:, 0], lse, o_ref, lse_ref, "decode many short", o_max_abs=bf16_arith_bound(_valid_vmax(c)))


def _valid_vmax(c):
    """Largest |V| entry among the sequences' own tokens (sentinel rows excluded)."""
    vmax = 0.0
    for b, L in enumerate(c.cache_seqlens.tolist()):
        if L == 0:
            continue
        t = torch.arange(L)
        rows = c.kv_pages[c.block_table[b, t // PAGE].long(), t % PAGE, 0, :DV]
        vmax = max(vmax, rows.float().abs().max().item())
    return vmax


def test_config5_full_size_sampled():
    """The bench workload in its launch configuration; the oracle recomputes
    a sample of sequences (all heads)."""
    c = inputs.decode_config_inputs()
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    rng = np.random.default_rng(5)
    seqs = sorted(set(rng.choice(64, size=6, replace=False).tolist()) |
                  {int(c.cache_seqlens.argmax()), int(c.cache_seqlens.argmin())})
    o_ref, lse_ref = _oracle(c, seqs)
    compare(o[seqs, 0], lse[seqs], o_ref, lse_ref, "MLA decode config")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    # |O| is bounded by the largest |V| entry among the sequences' own tokens
    assert o.float().abs().max().item() <= _valid_vmax(c) * (1 + 2 ** -7)


def test_deterministic_and_placement_invariant():
    lens = [700, 3000, 1, 129, 4100]
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=9)
    o1, l1 = _run(c)
    o2, l2 = _run(c)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # move every page to a new physical slot: the result must not change at all
    P = c.kv_pages.shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(3))
    pages2 = torch.empty_like(c.kv_pages)
    pages2[perm] = c.kv_pages
    c2 = inputs.PagedCache(c.q, pages2, perm[c.block_table.long()].to(torch.int32), c.cache_seqlens, PAGE)
    o3, l3 = _run(c2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_empty_sequences_give_zero_and_neg_inf():
    c = inputs.paged_decode_inputs(3, HQ, DK, [0, 10, 0], PAGE, seed=2)
    o, lse = _run(c)
    assert torch.all(o[0] == 0) and torch.all(o[2] == 0)
    assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isneginf(lse[2]))
    assert torch.isfinite(lse[1]).all()


def test_bad_block_table_entry_is_reported_not_read():
    c = inputs.paged_decode_inputs(2, HQ, DK, [100, 100], PAGE, seed=6)
    bt = c.block_table.clone()
    bt[1, 0] = c.kv_pages.shape[0] + 1000      # out of the pool
    c2 = inputs.PagedCache(c.q, c.kv_pages, bt, c.cache_seqlens, PAGE)
    _run(c2)
    assert ea.read_device_status(0) == 1      # ATTN_ERR_INVALID_ARG recorded on the device
    assert ea.read_device_status(0) == 0      # and cleared by the read


def test_workspace_checks():
    c = inputs.paged_decode_inputs(2, HQ, DK, [10, 20], PAGE, seed=1)
    q, kv, bt, sl = _dev(c)
    need = ea.decode_workspace_size(2, HQ, DV)
    assert need > 0
    lib = ea.library()
    # the size is that of the device named by the call's device argument
    assert lib.attn_decode_paged_workspace_size(2, HQ, DV, 0) == need
    assert lib.attn_decode_paged_workspace_size(2, HQ, DV, torch.cuda.device_count()) == 0
    assert lib.attn_decode_paged_workspace_size(2, HQ, DV, -1) == 0
    small = torch.empty(need - 256, dtype=torch.uint8, device=q.device)
    with pytest.raises(ValueError):
        ea.decode_paged(q, kv, bt, sl, SCALE, workspace=small)
    lib = ea.library()
    o = torch.empty((2, 1, HQ, DV), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((2, HQ), dtype=torch.float32, device=q.device)
    rc = lib.attn_decode_paged(q.data_ptr(), kv.data_ptr(), bt.data_ptr(), sl.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), 2, HQ, DK, DV, PAGE, kv.shape[0], bt.shape[1], SCALE,
                               small.data_ptr(), need - 256, None)
    assert rc == 5   # ATTN_ERR_WORKSPACE


def test_maximum_batch_of_sequences():
    """B = 2048, the largest batch the split plan holds in shared memory:
    2048 short sequences (0..40 tokens, so most pages are cut), checked on a
    sample of sequences against the oracle; the rest must be finite."""
    rng = np.random.default_rng(31)
    lens = rng.integers(0, 41, size=2048).tolist()
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=31)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    seqs = [0, 1, 511, 1024, 1500, 2047] + [int(np.argmax(lens))]
    o_ref, lse_ref = _oracle(c, seqs)
    compare(o[seqs, 0], lse[seqs], o_ref, lse_ref, "MLA decode B=2048", o_max_abs=bf16_arith_bound(_valid_vmax(c)))
    assert torch.isfinite(o).all()
    empty = torch.tensor(lens) == 0
    assert torch.isneginf(lse.cpu()[empty]).all() and torch.isfinite(lse.cpu()[~empty]).all()


def test_batch_above_maximum_is_rejected():
    c = inputs.paged_decode_inputs(2049, HQ, DK, [1] * 2049, PAGE, seed=2)
    with pytest.raises(ea.AttnError) as e:
        _run(c)
    assert e.value.code == 2
