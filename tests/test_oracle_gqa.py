"""Pins for the GQA-path paged-decode oracle (oracle.decode_paged_gqa).

What the function must compute ("GQLA: Group-Query Latent Attention ...", key
terms, GQA path: each group of query heads reads its own group-expanded cache;
"FlashMLA" page: 64-token pages reached through a block table;
"FlashAttention (KO)": softmax(scale * q K^T) V): query head h of sequence b
attends to the K and V rows of KV head h // (Hq / Hkv) of all L_b cached
tokens of that sequence.  Each pin below fixes that by something other than
the oracle itself: a pure-Python brute force, closed forms, the dense oracle
(pinned in test_oracle.py) on rows gathered with torch indexing, invariances,
and planted mistakes that must trip at least one pin.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_135_b200 import inputs

PAGE = 4


def _small(lens, Hq=4, Hkv=2, D=5, seed=7):
    return inputs.paged_gqa_decode_inputs(len(lens), Hq, Hkv, D, lens, PAGE, seed)


def _np(x):
    return x.to(torch.float64).numpy()


def _args(c):
    return (_np(c.q)[:, 0], _np(c.k_pages), _np(c.v_pages), c.block_table.numpy(), c.cache_seqlens.numpy())


def _brute(q, kp, vp, table, lens, scale, page):
    """Pure-Python loops with math.exp, one (sequence, head) at a time."""
    B, Hq, D = q.shape
    Hkv = kp.shape[2]
    O = [[[0.0] * D for _ in range(Hq)] for _ in range(B)]
    LSE = [[-math.inf] * Hq for _ in range(B)]
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            g = h // (Hq // Hkv)
            scores, rows = [], []
            for t in range(L):
                pg, r = int(table[b][t // page]), t % page
                s = 0.0
                for d in range(D):
                    s += float(q[b][h][d]) * float(kp[pg][r][g][d])
                scores.append(scale * s)
                rows.append([float(vp[pg][r][g][d]) for d in range(D)])
            if not scores:
                continue
            m = max(scores)
            w = [math.exp(s - m) for s in scores]
            tot = sum(w)
            for d in range(D):
                O[b][h][d] = sum(w[t] * rows[t][d] for t in range(L)) / tot
            LSE[b][h] = m + math.log(tot)
    return np.array(O), np.array(LSE)


def _check_brute(fn):
    c = _small([9, 0, 3, 4], Hq=4, Hkv=2, D=3)
    q, kp, vp, table, lens = _args(c)
    o, lse = fn(q, kp, vp, table, lens, 0.6, page_size=PAGE)
    ob, lb = _brute(q, kp, vp, table, lens, 0.6, PAGE)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


def test_brute_force():
    _check_brute(oracle.decode_paged_gqa)


def test_zero_query_gives_mean_of_group_values():
    c = _small([7, 12], Hq=6, Hkv=3, D=4)
    q, kp, vp, table, lens = _args(c)
    o, lse = oracle.decode_paged_gqa(np.zeros_like(q), kp, vp, table, lens, 0.9, page_size=PAGE)
    for b, L in enumerate(lens):
        t = torch.arange(int(L))
        for h in range(6):
            g = h // 2
            rows = c.v_pages[c.block_table[b, t // PAGE].long(), t % PAGE, g].to(torch.float64).numpy()
            np.testing.assert_allclose(o[b, h], rows.mean(0), atol=1e-13)
            assert abs(lse[b, h] - math.log(L)) < 1e-13


def test_single_token_returns_its_value():
    c = _small([1, 1], Hq=4, Hkv=4, D=6)
    q, kp, vp, table, lens = _args(c)
    o, lse = oracle.decode_paged_gqa(q, kp, vp, table, lens, 0.25, page_size=PAGE)
    for b in range(2):
        pg = int(table[b, 0])
        for h in range(4):
            np.testing.assert_allclose(o[b, h], vp[pg, 0, h], atol=1e-13)
            assert abs(lse[b, h] - 0.25 * float(q[b, h] @ kp[pg, 0, h])) < 1e-12


def test_equals_dense_oracle_on_gathered_rows():
    c = _small([13, 5, 22], Hq=8, Hkv=2, D=6)
    q, kp, vp, table, lens = _args(c)
    o, lse = oracle.decode_paged_gqa(q, kp, vp, table, lens, 0.4, page_size=PAGE)
    for b, L in enumerate(lens.tolist()):
        t = torch.arange(L)
        idx = c.block_table[b, t // PAGE].long()
        K = c.k_pages[idx, t % PAGE].to(torch.float64).numpy()        # [L, Hkv, D], torch gather
        V = c.v_pages[idx, t % PAGE].to(torch.float64).numpy()
        od, ld = oracle.attention(q[b][None, None], K[None], V[None], False, 0.4)
        np.testing.assert_allclose(o[b], od[0, 0], atol=1e-13)
        np.testing.assert_allclose(lse[b], ld[0, :, 0], atol=1e-13)


def test_invariant_to_page_placement_and_junk():
    c = _small([10, 3, 17])
    q, kp, vp, table, lens = _args(c)
    o1, l1 = oracle.decode_paged_gqa(q, kp, vp, table, lens, 0.5, page_size=PAGE)
    rng = np.random.default_rng(5)
    perm = rng.permutation(kp.shape[0])
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    table2 = perm[table]
    for b, L in enumerate(lens):
        npg = -(-int(L) // PAGE)
        if L % PAGE:
            kp2[table2[b, npg - 1], L % PAGE:] = 55.0
            vp2[table2[b, npg - 1], L % PAGE:] = -55.0
        table2[b, npg:] = table2[b, 0]
    o2, l2 = oracle.decode_paged_gqa(q, kp2, vp2, table2, lens, 0.5, page_size=PAGE)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_empty_sequence_and_subset():
    c = _small([0, 6, 2])
    q, kp, vp, table, lens = _args(c)
    o, lse = oracle.decode_paged_gqa(q, kp, vp, table, lens, 0.5, page_size=PAGE)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    o2, l2 = oracle.decode_paged_gqa(q, kp, vp, table, lens, 0.5, page_size=PAGE, seqs=[2, 1])
    np.testing.assert_allclose(o2, o[[2, 1]], atol=0)
    np.testing.assert_allclose(l2, lse[[2, 1]], atol=0)


def test_gqa_config_recipe():
    cfg = inputs.GQA_DECODE_CONFIG
    c = inputs.gqa_decode_config_inputs()
    lens = c.cache_seqlens
    assert lens.numel() == cfg.B and lens.min() >= cfg.min_len and lens.max() <= cfg.max_len
    npp = (lens + 63) // 64
    assert c.num_pages == int(npp.sum()) + 1
    used = torch.cat([c.block_table[b, :npp[b]] for b in range(cfg.B)])
    assert torch.equal(torch.sort(used).values, torch.arange(c.num_pages - 1, dtype=torch.int32))
    assert tuple(c.k_pages.shape[1:]) == (64, cfg.Hkv, cfg.D) and c.v_pages.shape == c.k_pages.shape
    poison = c.num_pages - 1
    assert torch.all(c.k_pages[poison].abs() == inputs.SENTINEL)
    # the tail rows of a cut last page hold sentinels, the rows before it do not
    b = int(torch.nonzero(lens % 64)[0])
    last = int(c.block_table[b, npp[b] - 1])
    r = int(lens[b] % 64)
    assert torch.all(c.v_pages[last, r:].abs() == inputs.SENTINEL)
    assert torch.all(c.v_pages[last, :r].abs() < inputs.SENTINEL)


# ---------------------------------------------------------------- planted mistakes (in the oracle, on the CPU)

def _mutant_wrong_group(q, kp, vp, table, lens, scale, page_size):
    # query head h reads KV head h % Hkv instead of h // group
    Hq, Hkv = q.shape[1], kp.shape[2]
    order = np.array([(g * (Hq // Hkv)) % Hkv for g in range(Hkv)])
    if np.array_equal(order, np.arange(Hkv)):
        order = order[::-1].copy()
    return oracle.decode_paged_gqa(q, kp[:, :, order], vp[:, :, order], table, lens, scale, page_size=page_size)


def _mutant_kv_swapped(q, kp, vp, table, lens, scale, page_size):
    return oracle.decode_paged_gqa(q, vp, kp, table, lens, scale, page_size=page_size)


def _mutant_no_scale(q, kp, vp, table, lens, scale, page_size):
    return oracle.decode_paged_gqa(q, kp, vp, table, lens, 1.0, page_size=page_size)


def _mutant_off_by_one_length(q, kp, vp, table, lens, scale, page_size):
    return oracle.decode_paged_gqa(q, kp, vp, table, np.maximum(np.asarray(lens) - 1, 0), scale, page_size=page_size)


@pytest.mark.parametrize("mutant", [_mutant_wrong_group, _mutant_kv_swapped, _mutant_no_scale,
                                    _mutant_off_by_one_length], ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(mutant):
    with pytest.raises(AssertionError):
        _check_brute(mutant)
