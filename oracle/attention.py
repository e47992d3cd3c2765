"""Plain fp64 CPU oracle for fused exact attention (test infrastructure only).

This module is test infrastructure.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it.  The CUDA library never calls it and shares no code with it.

What it computes is the plain definition the fused kernels must reach exactly
(up to rounding order):

* "FlashAttention (KO)", section "표준 Attention의 문제점" (the problem with
  standard attention): Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V.  The
  scale is a caller argument here (1/sqrt(d_k) in that formula; the MLA decode
  workload passes 1/sqrt(192)).
* "FlashAttention (KO)", section "온라인 Softmax 계산" (online softmax): the
  tiled method keeps a running max and a running exp-sum and still reaches the
  exact softmax result.  So the oracle does NOT tile: it materialises each full
  row of S = scale * Q K^T and applies the textbook softmax to it.
* "FlashAttention (KO)", section "단일 CUDA 커널로의 연산 융합" (fusion into one
  kernel): masking is one of the fused steps.  The only mask here is the causal
  one, aligned to the bottom-right corner: key j is visible to query i iff
  j <= i + (Nk - Nq).
* "GQLA: Group-Query Latent Attention ...", section 1 (MLA) and the
  "MQA-absorb path" definition: after absorption every query head attends to
  one shared latent KV row per token.  Here K is the whole 576-wide latent row
  and V is its first 512 entries.
* "FlashMLA" page, technical basis list: the KV cache is paged with 64-token
  pages; a block table maps each sequence's logical page to a physical page.
* "GQLA: Group-Query Latent Attention ...", key terms (GQA path): each group
  of query heads reads its own group-expanded cache.  Here that is a paged
  cache of separate K and V rows per (token, KV head); query head h reads KV
  head h // (Hq / Hkv), as in the dense oracle.
* "FlashAttention (KO)", section "FlashAttention-3 (2024)": FP8 inputs.  The
  page names no format; ``e4m3_decode`` follows the OCP 8-bit floating-point
  definition of E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits,
  subnormals at exponent field 0, no infinities, S.1111.111 is NaN), and
  ``attention_fp8`` is exact attention on the values the bytes represent.
* "Flash Attention" wiki page, section "구조화된 지식 (Synthesized Content)",
  item "Recomputation (재계산)": the backward pass recomputes the intermediate
  matrices instead of storing them.  ``attention_bwd`` writes out the plain
  derivative of the forward definition (dQ, dK, dV for an upstream dO).

Outputs: O (fp64) and LSE = ln sum_j exp(S_ij) (fp64, natural log of the sum
over the *scaled* scores).  A row with no visible key has O = 0, LSE = -inf.

Every value is computed in fp64 from the given input values (the bf16 inputs are
upcast exactly by the caller).  Row chunking below only bounds memory: each
chunk holds complete rows of S, so no online rescaling takes place.

Parity pins: tests/test_oracle.py checks this module against hand-derived
values (tests/golden/), closed forms, invariants, a pure-Python brute force
and torch's fp64 scaled_dot_product_attention; tests/test_oracle_gqa.py and
tests/test_oracle_mtp.py pin the GQA-path and multi-token decode functions
with brute forces, closed forms, invariances and planted mistakes;
tests/test_oracle_fp8.py pins the E4M3 decoding against torch's float8_e4m3fn,
hand-derived codes and planted mistakes;
tests/test_oracle_bwd.py pins the gradients with hand-derived cases
(tests/golden/hand_worked_bwd.json), central finite differences
of the forward function, torch fp64 autograd, closed forms, the zero sum of
the dK rows and planted mistakes.
"""

from __future__ import annotations

import numpy as np

__all__ = ["attention", "attention_bwd", "attention_fp8", "decode_paged", "decode_paged_mtp", "decode_paged_gqa",
           "e4m3_decode", "gather_pages"]


def _rows_softmax_weighted(S: np.ndarray, V: np.ndarray):
    """Textbook softmax of each row of S applied to V.

    Returns (O, LSE).  S holds -inf for masked entries.  Rows whose entries are
    all -inf give O = 0 and LSE = -inf (no visible key).
    """
    m = np.max(S, axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m_safe = np.where(np.isfinite(m), m, 0.0)
    P = np.exp(S - m_safe)                      # exp(-inf) = 0 for masked keys
    l = np.sum(P, axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        O = (P @ V) / l
        lse = m_safe[:, 0] + np.log(l[:, 0])
    O[empty] = 0.0
    lse[empty] = -np.inf
    return O, lse


def attention(q, k, v, causal: bool, scale: float, q_rows=None, row_chunk: int = 1024):
    """Exact attention, one (batch, query head) at a time, S materialised.

    q: [B, Nq, Hq, D]; k: [B, Nk, Hkv, D]; v: [B, Nk, Hkv, Dv] (any real dtype,
    upcast to fp64).  Query head hq reads KV head hq // (Hq // Hkv) (contiguous
    groups; grouped-query attention with Hkv = 1 is multi-query attention).

    q_rows: optional 1-D array of query row indices; only those rows are
    computed (for spot checks at full size).  Returns O [B, len(rows), Hq, Dv]
    and LSE [B, Hq, len(rows)] in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, Dk = k.shape
    Dv = v.shape[3]
    assert Dk == D and v.shape[:3] == (B, Nk, Hkv)
    assert Hq % Hkv == 0
    group = Hq // Hkv
    rows = np.arange(Nq) if q_rows is None else np.asarray(q_rows, dtype=np.int64)
    R = rows.shape[0]
    O = np.zeros((B, R, Hq, Dv), dtype=np.float64)
    LSE = np.full((B, Hq, R), -np.inf, dtype=np.float64)
    if Nk == 0 or R == 0:
        return O, LSE
    key_idx = np.arange(Nk)
    for b in range(B):
        for hq in range(Hq):
            kv = hq // group
            Kmat = k[b, :, kv, :]
            Vmat = v[b, :, kv, :]
            for c0 in range(0, R, row_chunk):
                r = rows[c0:c0 + row_chunk]
                S = scale * (q[b, r, hq, :] @ Kmat.T)
                if causal:
                    visible = key_idx[None, :] <= (r[:, None] + (Nk - Nq))
                    S = np.where(visible, S, -np.inf)
                o, lse = _rows_softmax_weighted(S, Vmat)
                O[b, c0:c0 + len(r), hq, :] = o
                LSE[b, hq, c0:c0 + len(r)] = lse
    return O, LSE


def gather_pages(kv_pages, block_table_row, seqlen: int, page_size: int):
    """Tokens 0..seqlen-1 of one sequence, read through its block-table row.

    kv_pages: [num_pages, page_size, Dk].  Token t lives in physical page
    block_table_row[t // page_size], row t % page_size.
    """
    kv_pages = np.asarray(kv_pages)
    out = np.empty((seqlen, kv_pages.shape[-1]), dtype=np.float64)
    for t0 in range(0, seqlen, page_size):
        page = int(block_table_row[t0 // page_size])
        n = min(page_size, seqlen - t0)
        out[t0:t0 + n] = kv_pages[page, :n, :]
    return out


def decode_paged(q, kv_pages, block_table, cache_seqlens, scale: float, dv: int,
                 page_size: int = 64, heads=None):
    """MLA absorbed decode over a paged latent cache (one query token per sequence).

    q: [B, Hq, Dk] absorbed queries; kv_pages: [num_pages, page_size, Dk] latent
    rows; block_table: [B, max_pages] int; cache_seqlens: [B] int.
    K = the gathered latent rows (all Dk entries), V = their first ``dv``
    entries; every query head attends to the same K/V (MQA-absorb form), no
    mask within the sequence (the single new token sees all cached tokens).
    heads: optional subset of query heads.  Returns O [B, len(heads), dv] and
    LSE [B, len(heads)] in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    kv_pages = np.asarray(kv_pages, dtype=np.float64)
    B, Hq, Dk = q.shape
    hs = np.arange(Hq) if heads is None else np.asarray(heads, dtype=np.int64)
    O = np.zeros((B, len(hs), dv), dtype=np.float64)
    LSE = np.full((B, len(hs)), -np.inf, dtype=np.float64)
    for b in range(B):
        L = int(cache_seqlens[b])
        if L == 0:
            continue
        Kmat = gather_pages(kv_pages, block_table[b], L, page_size)
        Vmat = Kmat[:, :dv]
        S = scale * (q[b, hs, :] @ Kmat.T)
        o, lse = _rows_softmax_weighted(S, Vmat)
        O[b] = o
        LSE[b] = lse
    return O, LSE


def decode_paged_gqa(q, k_pages, v_pages, block_table, cache_seqlens, scale: float, page_size: int = 64,
                     seqs=None):
    """GQA-path decode over a paged, group-expanded cache (one query token per sequence).

    q: [B, Hq, D]; k_pages, v_pages: [num_pages, page_size, Hkv, D];
    block_table: [B, max_pages] int; cache_seqlens: [B] int.  Query head h
    attends, with no mask inside the sequence, to the K and V rows of KV head
    h // (Hq // Hkv) of every cached token of its sequence.  seqs: optional
    subset of sequences.  Returns O [len(seqs), Hq, D] and LSE [len(seqs), Hq]
    in fp64; a sequence of length 0 gives O = 0 and LSE = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k_pages = np.asarray(k_pages, dtype=np.float64)
    v_pages = np.asarray(v_pages, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    group = Hq // Hkv
    bs = np.arange(B) if seqs is None else np.asarray(seqs, dtype=np.int64)
    O = np.zeros((len(bs), Hq, D), dtype=np.float64)
    LSE = np.full((len(bs), Hq), -np.inf, dtype=np.float64)
    for i, b in enumerate(bs):
        L = int(cache_seqlens[b])
        if L == 0:
            continue
        for g in range(Hkv):
            Kmat = gather_pages(k_pages[:, :, g, :], block_table[b], L, page_size)
            Vmat = gather_pages(v_pages[:, :, g, :], block_table[b], L, page_size)
            heads = np.arange(g * group, (g + 1) * group)
            S = scale * (q[b, heads, :] @ Kmat.T)
            o, lse = _rows_softmax_weighted(S, Vmat)
            O[i, heads] = o
            LSE[i, heads] = lse
    return O, LSE


def decode_paged_mtp(q, kv_pages, block_table, cache_seqlens, scale: float, dv: int, page_size: int = 64,
                     seqs=None):
    """MLA absorbed decode with s_q new query tokens per sequence.

    q: [B, s_q, Hq, Dk].  The s_q query tokens are the last s_q cached tokens
    of their sequence, so query token i of sequence b sees cached positions
    0 .. L_b - s_q + i: the causal mask aligned to the bottom-right corner of
    the dense formula (key j visible to query i iff j <= i + Nk - Nq, with
    Nq = s_q, Nk = L_b).  K = the gathered latent rows, V = their first dv
    entries, every head shares them (MQA-absorb form).  Returns O
    [len(seqs), s_q, Hq, dv] and LSE [len(seqs), s_q, Hq] in fp64; a query
    token with no visible position gets O = 0 and LSE = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    kv_pages = np.asarray(kv_pages, dtype=np.float64)
    B, sq, Hq, Dk = q.shape
    bs = np.arange(B) if seqs is None else np.asarray(seqs, dtype=np.int64)
    O = np.zeros((len(bs), sq, Hq, dv), dtype=np.float64)
    LSE = np.full((len(bs), sq, Hq), -np.inf, dtype=np.float64)
    for i, b in enumerate(bs):
        L = int(cache_seqlens[b])
        if L == 0:
            continue
        Kmat = gather_pages(kv_pages, block_table[b], L, page_size)
        o, lse = attention(q[b][None], Kmat[None, :, None, :], Kmat[None, :, None, :dv], True, scale)
        O[i] = o[0]
        LSE[i] = lse[0].T
    return O, LSE


def attention_bwd(q, k, v, do, causal: bool, scale: float, q_rows=None, k_rows=None, kv_heads=None,
                  row_chunk: int = 1024):
    """Gradients of exact attention with respect to Q, K and V.

    "Flash Attention" wiki page, section "구조화된 지식 (Synthesized Content)",
    item "Recomputation (재계산)": the backward pass does not keep the N x N
    intermediate matrices; it recomputes what it needs from the inputs.  The
    page gives no formulas.  What the backward must reach is the plain
    derivative of the forward definition (the one in ``attention``), which is
    what this function writes out, S and P materialised one block of complete
    rows at a time.  For one (batch, query head) with KV head kv and upstream
    gradient dO = dL/dO:

        S = scale * Q K^T (causal: -inf where key j > i + Nk - Nq)
        P = softmax of each row of S          (a row with no visible key: 0)
        dV_kv += P^T dO
        dP = dO V^T
        dS = P * (dP - rowsum(P * dP))          (softmax Jacobian, row by row)
        dQ = scale * dS K
        dK_kv += scale * dS^T Q

    dK and dV of a KV head sum over every query head of its group.

    q: [B, Nq, Hq, D]; k: [B, Nk, Hkv, D]; v: [B, Nk, Hkv, Dv]; do: [B, Nq, Hq, Dv].
    q_rows / k_rows: optional index arrays; dQ is returned for those query rows
    and dK, dV for those key rows only (every query row still enters dK and
    dV, so the cost stays that of the full problem).  kv_heads: optional
    subset of KV heads; only their query heads are computed, the other heads'
    entries stay 0.  Returns dQ [B, len(q_rows), Hq, D], dK [B, len(k_rows),
    Hkv, D], dV [B, len(k_rows), Hkv, Dv] in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    Dv = v.shape[3]
    assert do.shape == (B, Nq, Hq, Dv) and Hq % Hkv == 0
    group = Hq // Hkv
    qr = np.arange(Nq) if q_rows is None else np.asarray(q_rows, dtype=np.int64)
    kr = np.arange(Nk) if k_rows is None else np.asarray(k_rows, dtype=np.int64)
    heads_kv = range(Hkv) if kv_heads is None else [int(h) for h in kv_heads]
    dQ = np.zeros((B, len(qr), Hq, D))
    dK = np.zeros((B, len(kr), Hkv, D))
    dV = np.zeros((B, len(kr), Hkv, Dv))
    if Nk == 0 or Nq == 0:
        return dQ, dK, dV
    q_pos = {int(r): i for i, r in enumerate(qr)}
    key_idx = np.arange(Nk)
    for b in range(B):
        for kv in heads_kv:
            Kmat = k[b, :, kv, :]
            Vmat = v[b, :, kv, :]
            for hq in range(kv * group, (kv + 1) * group):
                for r0 in range(0, Nq, row_chunk):
                    rows = np.arange(r0, min(Nq, r0 + row_chunk))
                    S = scale * (q[b, rows, hq, :] @ Kmat.T)
                    if causal:
                        S = np.where(key_idx[None, :] <= rows[:, None] + (Nk - Nq), S, -np.inf)
                    m = np.max(S, axis=1, keepdims=True)
                    m = np.where(np.isfinite(m), m, 0.0)
                    E = np.exp(S - m)
                    l = np.sum(E, axis=1, keepdims=True)
                    P = np.divide(E, l, out=np.zeros_like(E), where=l > 0)
                    dOr = do[b, rows, hq, :]
                    dP = dOr @ Vmat.T
                    dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
                    dV[b, :, kv, :] += P[:, kr].T @ dOr
                    dK[b, :, kv, :] += scale * (dS[:, kr].T @ q[b, rows, hq, :])
                    sel = [i for i, r in enumerate(rows) if int(r) in q_pos]
                    if sel:
                        dQ[b, [q_pos[int(rows[i])] for i in sel], hq, :] = scale * (dS[sel] @ Kmat)
    return dQ, dK, dV


def e4m3_decode(codes):
    """Values of OCP FP8 E4M3 bytes, in fp64 (NaN for the two NaN codes).

    Bit layout s eeee mmm: exponent field e in 1..15 gives
    (-1)^s * 2^(e - 7) * (1 + m/8); e = 0 gives the subnormals
    (-1)^s * 2^-6 * (m/8); e = 15 with m = 7 is NaN (the format has no
    infinities, so 0x7E = 448 is the largest finite value).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = sign * np.ldexp(1.0 + m / 8.0, e - 7)
    sub = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, out)


def attention_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float, causal: bool, scale: float,
                  q_rows=None):
    """Exact attention on FP8 inputs: the definition of ``attention`` applied
    to the represented values descale * e4m3(byte), in fp64.

    q8 [B, Nq, Hq, D], k8 [B, Nk, Hkv, D], v8 [B, Nk, Hkv, D]: E4M3 bytes.
    Returns O and LSE as ``attention`` does.
    """
    q = q_descale * e4m3_decode(q8)
    k = k_descale * e4m3_decode(k8)
    v = v_descale * e4m3_decode(v8)
    return attention(q, k, v, causal, scale, q_rows=q_rows)
