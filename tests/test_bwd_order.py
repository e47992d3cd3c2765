"""Host logic of the backward's unit order (attn_bwd_head_group), on the CPU.

attn_bwd runs one CTA per (key block of 128, KV head, batch) and hands the
CTAs out g (batch, KV head) pairs at a time, key block slowest inside a
group.  The library takes g = ceil(SMs / key blocks) instead of all pairs
only when its model of the block scheduler (units in order to the SM that
frees first, each costing its query steps plus 4) gives at most 1 % more
makespan.  This test rebuilds that model independently (heapq) and checks the
library's choice against it on the shapes the rule was weighed on and on
random shapes, plus the fixed points: one pair, equal non-causal units,
rejected arguments.  The query needs no GPU.
"""

import heapq
import math
import random

import pytest

import exact_attention_135_b200 as ea

SMS = 148


def _model_choice(B, Hq, Hkv, Nq, Nk, D, causal, sms=SMS):
    bm = 64 if D == 128 else 128              # query rows per step of the kernel for D
    P, nkb, n_qblk, group = B * Hkv, -(-Nk // 128), -(-Nq // bm), Hq // Hkv
    g = min(P, -(-sms // nkb))
    if g >= P or P * nkb > (1 << 16):
        return P

    def steps(kb):
        first = max(0, math.trunc((kb * 128 - (Nk - Nq)) / bm)) if causal else 0
        return group * max(0, n_qblk - first) + 4

    def makespan(gs_max):
        free = [0] * sms
        end = 0
        for p0 in range(0, P, gs_max):
            for kb in range(nkb):
                for _ in range(min(gs_max, P - p0)):
                    t = heapq.heappop(free) + steps(kb)
                    heapq.heappush(free, t)
                    end = max(end, t)
        return end

    return g if makespan(g) * 100 <= makespan(P) * 101 else P


@pytest.mark.parametrize("shape, expect", [
    ((1, 32, 8, 16384, 16384, 128, True), 2),      # long-context GQA backward: two heads fill a wave
    ((4, 32, 8, 4096, 4096, 128, True), 32),       # grouping would start heavy blocks late
    ((2, 32, 4, 8192, 8192, 128, True), 8),
    ((4, 32, 8, 4096, 4096, 128, False), 5),       # equal units: grouping is free
    ((1, 32, 1, 16384, 16384, 128, True), 1),      # one pair
    ((1, 3, 3, 9600, 9600, 64, False), 2),         # the GPU test's shape: groups {0, 1}, {2}
    ((1, 3, 3, 9600, 9600, 128, False), 2),
    ((1, 2, 2, 300, 300, 64, True), 2),            # fewer key blocks than SMs: one wave
])
def test_choice_on_weighed_shapes(shape, expect):
    assert ea.bwd_head_group(*shape, SMS) == expect
    assert _model_choice(*shape) == expect


def test_choice_matches_independent_model_on_random_shapes():
    rng = random.Random(20261203)
    for _ in range(60):
        Hkv = rng.choice([1, 2, 4, 8])
        Hq = Hkv * rng.choice([1, 2, 4, 8])
        B = rng.choice([1, 2, 3, 4, 8])
        Nk = rng.choice([128, 1000, 4096, 8192, 9600, 16384, 20000])
        Nq = rng.choice([Nk, Nk // 2 + 1, 2 * Nk])
        D = rng.choice([64, 128])
        causal = rng.random() < 0.7
        got = ea.bwd_head_group(B, Hq, Hkv, Nq, Nk, D, causal, SMS)
        assert got == _model_choice(B, Hq, Hkv, Nq, Nk, D, causal), (B, Hq, Hkv, Nq, Nk, D, causal, got)
        assert 1 <= got <= B * Hkv


def test_rejected_arguments_give_zero():
    assert ea.bwd_head_group(1, 4, 2, 100, 0, 128, True, SMS) == 0       # no key blocks, no units
    assert ea.bwd_head_group(1, 3, 2, 100, 100, 128, True, SMS) == 0     # Hq not a multiple of Hkv
    assert ea.bwd_head_group(1, 4, 2, 100, 100, 256, True, SMS) == 0     # unsupported head dim
    assert ea.bwd_head_group(0, 4, 2, 100, 100, 128, True, SMS) == 0
    assert ea.bwd_head_group(1, 4, 2, 100, 100, 128, True, 0) == 0
