"""Pins for the multi-token MLA decode oracle (oracle.decode_paged_mtp).

What it must compute: s_q new query tokens per sequence, the last s_q
tokens of the cache, each attending causally to the cached positions up to
its own ("GQLA ..." page, MTP with the MQA-absorb path; "FlashAttention
(KO)": the formula, with the causal mask aligned to the bottom-right
corner).  Pinned by the single-token oracle on truncated lengths, a
pure-Python brute force, and planted mistakes.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_135_b200 import inputs

PAGE = 2


def _np(x):
    return x.to(torch.float64).numpy()


def _cache(lens, s_q, Hq=3, Dk=5, seed=3):
    return inputs.paged_decode_inputs(len(lens), Hq, Dk, lens, PAGE, seed, s_q=s_q)


def _args(c):
    return _np(c.q), _np(c.kv_pages)[:, :, 0], c.block_table.numpy(), c.cache_seqlens.numpy()


def _brute(q, pages, table, lens, scale, dv):
    B, sq, Hq, Dk = q.shape
    O = np.zeros((B, sq, Hq, dv))
    LSE = np.full((B, sq, Hq), -math.inf)
    for b in range(B):
        L = int(lens[b])
        for i in range(sq):
            last = L - sq + i           # last visible position
            for h in range(Hq):
                sc, rows = [], []
                for t in range(0, last + 1):
                    pg, r = int(table[b][t // PAGE]), t % PAGE
                    sc.append(scale * sum(float(q[b][i][h][d]) * float(pages[pg][r][d]) for d in range(Dk)))
                    rows.append([float(pages[pg][r][d]) for d in range(dv)])
                if not sc:
                    continue
                m = max(sc)
                w = [math.exp(x - m) for x in sc]
                tot = sum(w)
                for d in range(dv):
                    O[b, i, h, d] = sum(w[t] * rows[t][d] for t in range(len(w))) / tot
                LSE[b, i, h] = m + math.log(tot)
    return O, LSE


def _check_brute(fn):
    c = _cache([5, 2, 7], s_q=3, Hq=2, Dk=4)
    q, pages, table, lens = _args(c)
    o, lse = fn(q, pages, table, lens, 0.7, 3, page_size=PAGE)
    ob, lb = _brute(q, pages, table, lens, 0.7, 3)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


def test_brute_force_including_a_token_that_sees_nothing():
    _check_brute(oracle.decode_paged_mtp)


def test_single_token_equals_decode_paged():
    c = _cache([9, 4, 1], s_q=1)
    q, pages, table, lens = _args(c)
    o, lse = oracle.decode_paged_mtp(q, pages, table, lens, 0.4, 3, page_size=PAGE)
    o1, l1 = oracle.decode_paged(q[:, 0], pages, table, lens, 0.4, 3, page_size=PAGE)
    np.testing.assert_allclose(o[:, 0], o1, atol=1e-13)
    np.testing.assert_allclose(lse[:, 0], l1, atol=1e-13)


def test_token_i_equals_single_token_decode_of_truncated_sequence():
    c = _cache([11, 6, 4], s_q=4, Hq=4, Dk=6)
    q, pages, table, lens = _args(c)
    o, lse = oracle.decode_paged_mtp(q, pages, table, lens, 0.3, 5, page_size=PAGE)
    for i in range(4):
        cut = np.maximum(lens - 4 + 1 + i, 0)
        oi, li = oracle.decode_paged(q[:, i], pages, table, cut, 0.3, 5, page_size=PAGE)
        np.testing.assert_allclose(o[:, i], oi, atol=1e-13)
        np.testing.assert_allclose(lse[:, i], li, atol=1e-13)


def _mutant_no_mask(q, pages, table, lens, scale, dv, page_size):
    B, sq = q.shape[:2]
    outs = [oracle.decode_paged(q[:, i], pages, table, lens, scale, dv, page_size=page_size) for i in range(sq)]
    return np.stack([o for o, _ in outs], 1), np.stack([l for _, l in outs], 1)


def _mutant_top_left(q, pages, table, lens, scale, dv, page_size):
    B, sq = q.shape[:2]
    outs = [oracle.decode_paged(q[:, i], pages, table, np.minimum(lens, i + 1), scale, dv, page_size=page_size)
            for i in range(sq)]
    return np.stack([o for o, _ in outs], 1), np.stack([l for _, l in outs], 1)


@pytest.mark.parametrize("mutant", [_mutant_no_mask, _mutant_top_left], ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(mutant):
    with pytest.raises(AssertionError):
        _check_brute(mutant)
