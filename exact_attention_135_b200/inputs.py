"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds no attention arithmetic: it only draws tensors.  Both the
CUDA path and the fp64 oracle receive the values drawn here (the oracle gets
the same bf16 values upcast exactly to fp64).

Workloads (all inputs i.i.d. N(0,1), drawn in fp32 from a CPU generator seeded
with 1000 + workload number, then rounded to bf16):

1. tiny exact attention: B=1, H=2, Nq=Nk=128, D=64, non-causal, scale 1/8.
2. GPT-2-small-shaped causal prefill: B=8, Hq=Hkv=12, N=1024, D=64.
3. long-context GQA causal prefill: B=1, Hq=32, Hkv=8, N=16384, D=128.
4. MQA wide-head non-causal: B=4, Hq=16, Hkv=1, N=4096, D=256, Q doubled
   before rounding (exact in bf16) for peaked softmax rows.
5. MLA absorbed paged decode: 64 sequences x 1 query token x 128 heads, one
   576-wide latent row per token (K = all 576, V = first 512), 64-token pages,
   lengths uniform on [1024, 8192], block table = a random permutation of the
   page pool, scale 1/sqrt(192).
6. GQA-path paged decode: 64 sequences x 1 query token x 32 query heads in 8
   groups of 4, each group reading its own expanded K and V rows (D=128) from
   64-token pages; lengths uniform on [1024, 8192], random page permutation,
   scale 1/sqrt(128).  The head geometry is LLaMA-3-8B's (the GQA model the
   GQLA page converts); the pages give no decode shapes for this path.

Paged-cache layout (decode): the pool holds exactly sum_b ceil(L_b/64) pages
plus one poison page at the end.  Block-table entries past a sequence's last
page point at the poison page.  Rows of a last page beyond L_b, and the whole
poison page, hold large finite values (+-1024): a kernel that reads them by
mistake produces a gross numeric error rather than a silent one, and since
they are finite a correct kernel that multiplies them by a zero weight is
unaffected.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

PAGE_SIZE = 64
SENTINEL = 1024.0


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    Dv: int
    causal: bool
    scale: float
    q_mult: float = 1.0
    seed: int = 0

    def flops(self) -> float:
        """4*Nq*Nk*D per (batch, query head), halved when causal (Nq == Nk)."""
        f = 4.0 * self.Nq * self.Nk * self.D * self.B * self.Hq
        return f / 2.0 if self.causal else f

    def io_bytes(self) -> int:
        """Compulsory HBM bytes: read Q, K, V once, write O (bf16) and LSE (fp32)."""
        q = self.B * self.Nq * self.Hq * self.D * 2
        k = self.B * self.Nk * self.Hkv * self.D * 2
        v = self.B * self.Nk * self.Hkv * self.Dv * 2
        o = self.B * self.Nq * self.Hq * self.Dv * 2
        lse = self.B * self.Hq * self.Nq * 4
        return q + k + v + o + lse


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    Hq: int
    Dk: int
    Dv: int
    page_size: int
    min_len: int
    max_len: int
    scale: float
    seed: int = 0


PREFILL_CONFIGS = {
    1: PrefillConfig("tiny B1 H2 N128 D64", 1, 2, 2, 128, 128, 64, 64, False, 1.0 / 8.0, seed=1001),
    2: PrefillConfig("gpt2-small causal B8 H12 N1024 D64", 8, 12, 12, 1024, 1024, 64, 64, True,
                     1.0 / 8.0, seed=1002),
    3: PrefillConfig("long GQA causal B1 Hq32 Hkv8 N16384 D128", 1, 32, 8, 16384, 16384, 128, 128, True,
                     1.0 / math.sqrt(128.0), seed=1003),
    4: PrefillConfig("MQA wide-head B4 Hq16 Hkv1 N4096 D256", 4, 16, 1, 4096, 4096, 256, 256, False,
                     1.0 / 16.0, q_mult=2.0, seed=1004),
}

DECODE_CONFIG = DecodeConfig("MLA absorbed paged decode B64 Hq128 Dk576 Dv512 page64", 64, 128, 576, 512,
                             PAGE_SIZE, 1024, 8192, 1.0 / math.sqrt(192.0), seed=1005)


def _randn_bf16(gen: torch.Generator, shape, mult: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if mult != 1.0:
        x = x * mult
    return x.to(torch.bfloat16)


def prefill_inputs(B, Hq, Hkv, Nq, Nk, D, Dv, seed, q_mult=1.0):
    """Q [B,Nq,Hq,D], K [B,Nk,Hkv,D], V [B,Nk,Hkv,Dv] bf16 CPU tensors, contiguous."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    q = _randn_bf16(gen, (B, Nq, Hq, D), q_mult)
    k = _randn_bf16(gen, (B, Nk, Hkv, D))
    v = _randn_bf16(gen, (B, Nk, Hkv, Dv))
    return q, k, v


def prefill_config_inputs(cfg: PrefillConfig):
    return prefill_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.Dv, cfg.seed, cfg.q_mult)


E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor FP8 (E4M3) encoding of an fp32 tensor for the FP8 forward.

    descale = max|x| / 448, rounded to fp32 (the value both the kernel and
    the oracle then use); the bytes are x / descale rounded to nearest even
    by torch's float8_e4m3fn cast, returned as uint8.  Returns (bytes, descale).
    """
    amax = float(x.abs().max()) if x.numel() else 0.0
    descale = float(torch.tensor(amax / E4M3_MAX if amax > 0 else 1.0, dtype=torch.float32))
    q = (x / descale).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), descale


def fp8_prefill_inputs(B, Hq, Hkv, Nq, Nk, D, seed, q_mult=1.0):
    """FP8 forward inputs: Q, K, V drawn as prefill_inputs draws them (the same
    generator stream, kept in fp32 instead of rounded to bf16), then each
    encoded per tensor by quantize_e4m3.  Returns (q8, k8, v8, (dq, dk, dv))."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    q = torch.randn(B, Nq, Hq, D, generator=gen, dtype=torch.float32) * q_mult
    k = torch.randn(B, Nk, Hkv, D, generator=gen, dtype=torch.float32)
    v = torch.randn(B, Nk, Hkv, D, generator=gen, dtype=torch.float32)
    (q8, dq), (k8, dk), (v8, dv) = quantize_e4m3(q), quantize_e4m3(k), quantize_e4m3(v)
    return q8, k8, v8, (dq, dk, dv)


def bwd_inputs(B, Hq, Hkv, Nq, Nk, D, seed, q_mult=1.0):
    """Backward-pass inputs: Q, K, V exactly as prefill_inputs draws them for
    the same seed, plus the upstream gradient dO [B,Nq,Hq,D] ~ N(0,1) in bf16
    from a second generator seeded seed + 7919."""
    q, k, v = prefill_inputs(B, Hq, Hkv, Nq, Nk, D, D, seed, q_mult)
    gen = torch.Generator(device="cpu").manual_seed(int(seed) + 7919)
    do = _randn_bf16(gen, (B, Nq, Hq, D))
    return q, k, v, do


def bwd_config_inputs(cfg: PrefillConfig):
    return bwd_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nk, cfg.D, cfg.seed, cfg.q_mult)


@dataclass
class PagedCache:
    q: torch.Tensor              # [B, 1, Hq, Dk] bf16
    kv_pages: torch.Tensor       # [num_pages, page_size, 1, Dk] bf16 (last page = poison)
    block_table: torch.Tensor    # [B, max_pages_per_seq] int32
    cache_seqlens: torch.Tensor  # [B] int32
    page_size: int

    @property
    def num_pages(self) -> int:
        return int(self.kv_pages.shape[0])

    def kv_valid_bytes(self, dk: int) -> int:
        """Bytes of latent rows that belong to the sequences (what a decode step must read)."""
        return int(self.cache_seqlens.to(torch.int64).sum()) * dk * 2


def paged_decode_inputs(B, Hq, Dk, seqlens, page_size, seed, max_pages_per_seq=None, s_q=1):
    """Build a paged latent cache for the given sequence lengths.

    seqlens: list/1-D tensor of lengths (0 allowed).  s_q: query tokens per
    sequence (q is [B, s_q, Hq, Dk]).  Returns a PagedCache.
    """
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).reshape(-1)
    assert seqlens.numel() == B
    pages_per_seq = [(int(L) + page_size - 1) // page_size for L in seqlens.tolist()]
    n_used = sum(pages_per_seq)
    max_pp = max(pages_per_seq + [1]) if max_pages_per_seq is None else int(max_pages_per_seq)
    poison = n_used                      # index of the poison page
    q = _randn_bf16(gen, (B, s_q, Hq, Dk))
    pool = _randn_bf16(gen, (n_used + 1, page_size, 1, Dk))
    sign = torch.randint(0, 2, (n_used + 1, page_size, 1, Dk), generator=gen) * 2 - 1
    sentinel = (sign.to(torch.float32) * SENTINEL).to(torch.bfloat16)
    pool[poison] = sentinel[poison]
    perm = torch.randperm(n_used, generator=gen).to(torch.int32)
    table = torch.full((B, max_pp), poison, dtype=torch.int32)
    cursor = 0
    for b, npg in enumerate(pages_per_seq):
        table[b, :npg] = perm[cursor:cursor + npg]
        cursor += npg
        L = int(seqlens[b])
        if npg and L % page_size:
            last = int(table[b, npg - 1])
            pool[last, L % page_size:] = sentinel[last, L % page_size:]
    return PagedCache(q, pool, table, seqlens.clone(), page_size)


@dataclass(frozen=True)
class GqaDecodeConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    min_len: int
    max_len: int
    scale: float
    seed: int = 0


GQA_DECODE_CONFIG = GqaDecodeConfig("GQA-path paged decode B64 Hq32 Hkv8 D128 page64", 64, 32, 8, 128, PAGE_SIZE,
                                    1024, 8192, 1.0 / math.sqrt(128.0), seed=1006)


@dataclass
class PagedKV:
    q: torch.Tensor              # [B, 1, Hq, D] bf16
    k_pages: torch.Tensor        # [num_pages, page_size, Hkv, D] bf16 (last page = poison)
    v_pages: torch.Tensor        # [num_pages, page_size, Hkv, D] bf16 (last page = poison)
    block_table: torch.Tensor    # [B, max_pages_per_seq] int32
    cache_seqlens: torch.Tensor  # [B] int32
    page_size: int

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    def kv_valid_bytes(self) -> int:
        """Bytes of K and V rows that belong to the sequences (what a decode step must read)."""
        hkv, d = int(self.k_pages.shape[2]), int(self.k_pages.shape[3])
        return int(self.cache_seqlens.to(torch.int64).sum()) * hkv * d * 2 * 2


def paged_gqa_decode_inputs(B, Hq, Hkv, D, seqlens, page_size, seed, max_pages_per_seq=None):
    """Build separate K and V page pools (GQA path: one expanded K and V row per
    token and KV head) for the given sequence lengths.  Same pool, poison-page
    and block-table conventions as paged_decode_inputs.  Returns a PagedKV."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).reshape(-1)
    assert seqlens.numel() == B
    pages_per_seq = [(int(L) + page_size - 1) // page_size for L in seqlens.tolist()]
    n_used = sum(pages_per_seq)
    max_pp = max(pages_per_seq + [1]) if max_pages_per_seq is None else int(max_pages_per_seq)
    poison = n_used
    q = _randn_bf16(gen, (B, 1, Hq, D))
    k_pool = _randn_bf16(gen, (n_used + 1, page_size, Hkv, D))
    v_pool = _randn_bf16(gen, (n_used + 1, page_size, Hkv, D))

    def sentinel(shape):
        sign = torch.randint(0, 2, shape, generator=gen, dtype=torch.int16) * 2 - 1
        return (sign.to(torch.float32) * SENTINEL).to(torch.bfloat16)

    k_pool[poison] = sentinel(k_pool[poison].shape)
    v_pool[poison] = sentinel(v_pool[poison].shape)
    perm = torch.randperm(n_used, generator=gen).to(torch.int32)
    table = torch.full((B, max_pp), poison, dtype=torch.int32)
    cursor = 0
    for b, npg in enumerate(pages_per_seq):
        table[b, :npg] = perm[cursor:cursor + npg]
        cursor += npg
        L = int(seqlens[b])
        if npg and L % page_size:
            last = int(table[b, npg - 1])
            k_pool[last, L % page_size:] = sentinel(k_pool[last, L % page_size:].shape)
            v_pool[last, L % page_size:] = sentinel(v_pool[last, L % page_size:].shape)
    return PagedKV(q, k_pool, v_pool, table, seqlens.clone(), page_size)


def gqa_decode_config_inputs(cfg: GqaDecodeConfig = GQA_DECODE_CONFIG):
    gen = torch.Generator(device="cpu").manual_seed(int(cfg.seed))
    seqlens = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.B,), generator=gen, dtype=torch.int32)
    return paged_gqa_decode_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, seqlens, cfg.page_size, cfg.seed + 100000)


def decode_config_inputs(cfg: DecodeConfig = DECODE_CONFIG):
    gen = torch.Generator(device="cpu").manual_seed(int(cfg.seed))
    seqlens = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.B,), generator=gen, dtype=torch.int32)
    return paged_decode_inputs(cfg.B, cfg.Hq, cfg.Dk, seqlens, cfg.page_size, cfg.seed + 100000)
