"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself: hand-derived values
(tests/golden/hand_worked.json), closed forms, invariants of the softmax
definition, a pure-Python brute force on tiny inputs, and torch's fp64
scaled_dot_product_attention.  The last test plants mistakes in copies of the
oracle and checks that the pins catch each one.
"""

import json
import math
import os
import re

import numpy as np
import pytest
import torch

import oracle

from exact_attention_135_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _val(x):
    if isinstance(x, (int, float)):
        return float(x)
    s = x.strip()
    if s == "-inf":
        return -math.inf
    m = re.fullmatch(r"ln(\d+)(?:/(\d+))?", s)
    if m:
        v = math.log(int(m.group(1)))
        return v / int(m.group(2)) if m.group(2) else v
    return float(s)


def _arr(nested):
    return np.vectorize(_val, otypes=[np.float64])(np.array(nested, dtype=object))


with open(GOLDEN) as f:
    _G = json.load(f)


@pytest.mark.parametrize("case", _G["prefill"], ids=[c["name"] for c in _G["prefill"]])
def test_hand_worked_prefill(case):
    q, k, v = _arr(case["q"]), _arr(case["k"]), _arr(case["v"])
    o, lse = oracle.attention(q, k, v, case["causal"], case["scale"])
    np.testing.assert_allclose(o, _arr(case["o"]), rtol=0, atol=1e-14)
    exp_lse = _arr(case["lse"])
    assert np.array_equal(np.isneginf(lse), np.isneginf(exp_lse))
    fin = np.isfinite(exp_lse)
    np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", _G["decode"], ids=[c["name"] for c in _G["decode"]])
def test_hand_worked_decode(case):
    q = _arr(case["q"])
    pages = _arr(case["kv_pages"])
    o, lse = oracle.decode_paged(q, pages, np.array(case["block_table"]), np.array(case["cache_seqlens"]),
                                 case["scale"], case["dv"], page_size=case["page_size"])
    np.testing.assert_allclose(o, _arr(case["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, _arr(case["lse"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- brute force

def _brute(q, k, v, causal, scale):
    """Pure-Python loops with math.exp: the formula written out term by term."""
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    Dv = v.shape[3]
    g = Hq // Hkv
    O = np.zeros((B, Nq, Hq, Dv))
    L = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i in range(Nq):
                scores = []
                for j in range(Nk):
                    if causal and j > i + (Nk - Nq):
                        continue
                    s = 0.0
                    for d in range(D):
                        s += float(q[b, i, h, d]) * float(k[b, j, kh, d])
                    scores.append((j, scale * s))
                if not scores:
                    L[b, h, i] = -math.inf
                    continue
                mx = max(s for _, s in scores)
                w = [(j, math.exp(s - mx)) for j, s in scores]
                tot = sum(x for _, x in w)
                for d in range(Dv):
                    O[b, i, h, d] = sum(x * float(v[b, j, kh, d]) for j, x in w) / tot
                L[b, h, i] = mx + math.log(tot)
    return O, L


BRUTE_CASES = [
    # (B, Nq, Nk, Hq, Hkv, D, Dv, causal)
    (1, 4, 4, 1, 1, 4, 4, False),
    (1, 4, 4, 1, 1, 4, 4, True),
    (1, 3, 5, 2, 1, 3, 2, True),
    (1, 5, 3, 2, 2, 2, 3, True),
    (2, 4, 6, 4, 2, 3, 3, False),
]


@pytest.mark.parametrize("shape", BRUTE_CASES)
def test_brute_force(shape):
    B, Nq, Nk, Hq, Hkv, D, Dv, causal = shape
    rng = np.random.default_rng(sum(shape[:7]))
    q = rng.standard_normal((B, Nq, Hq, D))
    k = rng.standard_normal((B, Nk, Hkv, D))
    v = rng.standard_normal((B, Nk, Hkv, Dv))
    scale = 0.7
    o, lse = oracle.attention(q, k, v, causal, scale)
    ob, lb = _brute(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_zero_query_gives_uniform_weights():
    rng = np.random.default_rng(1)
    B, N, H, D = 1, 7, 2, 5
    q = np.zeros((B, N, H, D))
    k = rng.standard_normal((B, N, H, D))
    v = rng.standard_normal((B, N, H, D))
    o, lse = oracle.attention(q, k, v, False, 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(N), atol=1e-14)
    oc, lsec = oracle.attention(q, k, v, True, 0.3)
    prefix = np.cumsum(v, axis=1) / np.arange(1, N + 1)[None, :, None, None]
    np.testing.assert_allclose(oc, prefix, atol=1e-14)
    np.testing.assert_allclose(lsec, np.log(np.arange(1, N + 1))[None, None, :].repeat(H, 1), atol=1e-14)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 5, 3, 4))
    k = rng.standard_normal((2, 1, 3, 4))
    v = rng.standard_normal((2, 1, 3, 6))
    o, lse = oracle.attention(q, k, v, False, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("bnhd,bhd->bhn", q, k[:, 0]), atol=1e-13)


def test_causal_row0_is_v0():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 6, 2, 4))
    k = rng.standard_normal((1, 6, 2, 4))
    v = rng.standard_normal((1, 6, 2, 4))
    o, lse = oracle.attention(q, k, v, True, 0.8)
    np.testing.assert_allclose(o[:, 0], v[:, 0], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], 0.8 * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]), atol=1e-14)


def test_constant_value_row():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 9, 2, 4))
    k = rng.standard_normal((1, 9, 2, 4))
    row = rng.standard_normal(5)
    v = np.broadcast_to(row, (1, 9, 2, 5)).copy()
    for causal in (False, True):
        o, _ = oracle.attention(q, k, v, causal, 1.3)
        np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), atol=1e-13)


# ---------------------------------------------------------------- invariants

def test_softmax_rows_sum_to_one():
    # With V = identity over the keys, O is exactly the weight matrix P.
    rng = np.random.default_rng(5)
    N = 6
    q = rng.standard_normal((1, N, 1, 3))
    k = rng.standard_normal((1, N, 1, 3))
    v = np.eye(N)[None, :, None, :]
    for causal in (False, True):
        P, _ = oracle.attention(q, k, v, causal, 2.0)
        P = P[0, :, 0, :]
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
        assert (P >= 0).all()
        if causal:
            assert np.all(P[np.triu_indices(N, 1)] == 0.0)


def test_key_permutation_invariance():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((2, 5, 2, 4))
    k = rng.standard_normal((2, 11, 2, 4))
    v = rng.standard_normal((2, 11, 2, 3))
    perm = rng.permutation(11)
    o1, l1 = oracle.attention(q, k, v, False, 0.6)
    o2, l2 = oracle.attention(q, k[:, perm], v[:, perm], False, 0.6)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(7)
    Hq, Hkv = 6, 2
    q = rng.standard_normal((1, 8, Hq, 4))
    k = rng.standard_normal((1, 8, Hkv, 4))
    v = rng.standard_normal((1, 8, Hkv, 4))
    o1, l1 = oracle.attention(q, k, v, True, 0.5)
    krep = np.repeat(k, Hq // Hkv, axis=2)
    vrep = np.repeat(v, Hq // Hkv, axis=2)
    o2, l2 = oracle.attention(q, krep, vrep, True, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)


def test_split_merge_identity():
    """Partials over disjoint key ranges, merged by their LSEs, equal the full result.

    lse = ln sum_i exp(lse_i), O = sum_i exp(lse_i - lse) O_i: the algebra behind
    the running max / running sum of the online softmax ("FlashAttention (KO)",
    online softmax section), and behind the split-KV combine step.
    """
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 3, 2, 5))
    k = rng.standard_normal((1, 13, 2, 5))
    v = rng.standard_normal((1, 13, 2, 4))
    o, lse = oracle.attention(q, k, v, False, 0.9)
    cuts = [0, 4, 5, 13]
    parts = [oracle.attention(q, k[:, a:b], v[:, a:b], False, 0.9) for a, b in zip(cuts[:-1], cuts[1:])]
    lses = np.stack([p[1] for p in parts])                      # [parts, B, H, Nq]
    lse_m = np.log(np.sum(np.exp(lses), axis=0))
    w = np.exp(lses - lse_m)                                     # [parts, B, H, Nq]
    o_m = sum(np.transpose(w[i], (0, 2, 1))[..., None] * parts[i][0] for i in range(len(parts)))
    np.testing.assert_allclose(lse_m, lse, atol=1e-12)
    np.testing.assert_allclose(o_m, o, atol=1e-12)


def test_row_subset_matches_full():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 37, 4, 8))
    k = rng.standard_normal((2, 37, 2, 8))
    v = rng.standard_normal((2, 37, 2, 8))
    o, lse = oracle.attention(q, k, v, True, 0.35, row_chunk=5)
    rows = np.array([0, 3, 17, 36])
    os_, ls = oracle.attention(q, k, v, True, 0.35, q_rows=rows)
    np.testing.assert_allclose(os_, o[:, rows], atol=1e-14)
    np.testing.assert_allclose(ls, lse[:, :, rows], atol=1e-14)


# ---------------------------------------------------------------- library cross-check

@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(causal):
    rng = np.random.default_rng(10)
    B, N, H, D = 2, 33, 3, 16
    q = rng.standard_normal((B, N, H, D))
    k = rng.standard_normal((B, N, H, D))
    v = rng.standard_normal((B, N, H, D))
    o, _ = oracle.attention(q, k, v, causal, 0.25)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal, scale=0.25)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


# ---------------------------------------------------------------- paged decode

def _small_cache(seqlens, seed=11, Hq=4, Dk=24, page=8):
    return inputs.paged_decode_inputs(len(seqlens), Hq, Dk, seqlens, page, seed)


def _np(x):
    return x.to(torch.float64).numpy()


def test_decode_equals_dense_on_gathered_tokens():
    c = _small_cache([17, 8, 1, 30])
    dv = 16
    q = _np(c.q)[:, 0]
    pages = _np(c.kv_pages)[:, :, 0]
    o, lse = oracle.decode_paged(q, pages, c.block_table.numpy(), c.cache_seqlens.numpy(), 0.3, dv, page_size=8)
    for b, L in enumerate(c.cache_seqlens.tolist()):
        # gather with torch indexing (independent of the oracle's loop)
        t = torch.arange(L)
        rows = c.kv_pages[c.block_table[b, t // 8].long(), t % 8, 0].to(torch.float64).numpy()
        od, ld = oracle.attention(q[b][None, None], rows[None, :, None, :], rows[None, :, None, :dv], False, 0.3)
        np.testing.assert_allclose(o[b], od[0, 0], atol=1e-13)
        np.testing.assert_allclose(lse[b], ld[0, :, 0], atol=1e-13)


def test_decode_invariant_to_page_placement_and_poison():
    c = _small_cache([19, 40, 3])
    q = _np(c.q)[:, 0]
    pages = _np(c.kv_pages)[:, :, 0]
    table = c.block_table.numpy()
    lens = c.cache_seqlens.numpy()
    o1, l1 = oracle.decode_paged(q, pages, table, lens, 0.4, 10, page_size=8)
    rng = np.random.default_rng(12)
    perm = rng.permutation(pages.shape[0])           # new physical slot of each page
    pages2 = np.empty_like(pages)
    pages2[perm] = pages
    table2 = perm[table]
    # overwrite everything a sequence must not read with other finite junk
    for b, L in enumerate(lens):
        npg = -(-L // 8)
        if L % 8:
            pages2[table2[b, npg - 1], L % 8:] = -77.0
        table2[b, npg:] = table2[b, 0]
    o2, l2 = oracle.decode_paged(q, pages2, table2, lens, 0.4, 10, page_size=8)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_decode_empty_sequence():
    c = _small_cache([0, 5])
    o, lse = oracle.decode_paged(_np(c.q)[:, 0], _np(c.kv_pages)[:, :, 0], c.block_table.numpy(),
                                 c.cache_seqlens.numpy(), 0.5, 8, page_size=8)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


# ---------------------------------------------------------------- inputs recipe

def test_input_recipe_properties():
    c = inputs.decode_config_inputs()
    lens = c.cache_seqlens
    assert lens.min() >= 1024 and lens.max() <= 8192 and lens.numel() == 64
    npp = (lens + 63) // 64
    assert c.num_pages == int(npp.sum()) + 1
    used = torch.cat([c.block_table[b, :npp[b]] for b in range(64)])
    assert torch.equal(torch.sort(used).values, torch.arange(c.num_pages - 1, dtype=torch.int32))
    q, k, v = inputs.prefill_inputs(1, 2, 2, 128, 128, 64, 64, 1001)
    q2, _, _ = inputs.prefill_inputs(1, 2, 2, 128, 128, 64, 64, 1001)
    assert torch.equal(q, q2) and q.dtype == torch.bfloat16


# ---------------------------------------------------------------- planted mistakes

def _mutants():
    base = oracle.attention

    def no_scale(q, k, v, causal, scale, **kw):
        return base(q, k, v, causal, 1.0, **kw)

    def top_left_causal(q, k, v, causal, scale, **kw):
        # wrong alignment: j <= i instead of j <= i + Nk - Nq
        q = np.asarray(q, dtype=np.float64)
        if causal and q.shape[1] != k.shape[1]:
            Nq, Nk = q.shape[1], k.shape[1]
            pad = np.zeros((q.shape[0], Nk - Nq, q.shape[2], q.shape[3])) if Nk > Nq else None
            if pad is not None:
                o, l = base(np.concatenate([q, pad], 1), k, v, causal, scale)
                return o[:, :Nq], l[:, :, :Nq]
        return base(q, k, v, causal, scale, **kw)

    def wrong_group(q, k, v, causal, scale, **kw):
        k = np.asarray(k)
        v = np.asarray(v)
        Hq, Hkv = np.asarray(q).shape[2], k.shape[2]
        if Hkv > 1 and Hq != Hkv:
            idx = np.arange(Hq) % Hkv
            return base(q, k[:, :, idx], v[:, :, idx], causal, scale, **kw)
        return base(q, k, v, causal, scale, **kw)

    def transposed_v(q, k, v, causal, scale, **kw):
        v = np.asarray(v)
        return base(q, k, v[:, ::-1], causal, scale, **kw)

    def log2_lse(q, k, v, causal, scale, **kw):
        o, l = base(q, k, v, causal, scale, **kw)
        return o, l / math.log(2.0)

    return [no_scale, top_left_causal, wrong_group, transposed_v, log2_lse]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    monkeypatch.setattr(oracle, "attention", mutant)
    failures = 0
    checks = [lambda c=c: test_hand_worked_prefill(c) for c in _G["prefill"]]
    checks += [lambda s=s: _brute_check(mutant, s) for s in BRUTE_CASES]
    for chk in checks:
        try:
            chk()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught mutant {mutant.__name__}"


def _brute_check(fn, shape):
    B, Nq, Nk, Hq, Hkv, D, Dv, causal = shape
    rng = np.random.default_rng(sum(shape[:7]))
    q = rng.standard_normal((B, Nq, Hq, D))
    k = rng.standard_normal((B, Nk, Hkv, D))
    v = rng.standard_normal((B, Nk, Hkv, Dv))
    o, lse = fn(q, k, v, causal, 0.7)
    ob, lb = _brute(q, k, v, causal, 0.7)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)
