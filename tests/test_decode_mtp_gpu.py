"""GPU parity of attn_decode_paged_mtp (s_q query tokens per sequence, MLA
absorbed paged decode, through the C ABI) against the fp64 oracle."""

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


def _run(c):
    d = torch.device("cuda:0")
    o, lse = ea.decode_paged_mtp(c.q.to(d), c.kv_pages.to(d), c.block_table.to(d), c.cache_seqlens.to(d), SCALE,
                                 dv=DV)
    torch.cuda.synchronize()
    return o, lse


def _oracle(c, seqs=None):
    return oracle.decode_paged_mtp(to_np64(c.q), to_np64(c.kv_pages)[:, :, 0], c.block_table.numpy(),
                                   c.cache_seqlens.numpy(), SCALE, DV, page_size=PAGE, seqs=seqs)


def _vmax(c):
    m = 0.0
    for b, L in enumerate(c.cache_seqlens.tolist()):
        t = torch.arange(L)
        if L:
            m = max(m, float(c.kv_pages[c.block_table[b, t // PAGE].long(), t % PAGE, 0, :DV].abs().max()))
    return m


@pytest.mark.parametrize("lens,s_q", [
    ([1], 2),                    # the first token sees nothing
    ([64, 65, 2], 2),            # the second token crosses a page boundary
    ([300, 0, 1000, 3], 3),
    ([8192], 4),                 # one long sequence split over every CTA pair
    ([5000, 17, 4096, 64 * 37], 2),
])
def test_small_batches(lens, s_q):
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=sum(lens) + s_q, s_q=s_q)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    o_ref, lse_ref = _oracle(c)
    compare(o, lse, o_ref, lse_ref, f"mtp decode s_q={s_q} lens={lens}", o_max_abs=bf16_arith_bound(_vmax(c)))


def test_single_token_matches_decode_paged_bitwise():
    lens = [700, 64, 3000]
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=8, s_q=1)
    o1, l1 = _run(c)
    d = torch.device("cuda:0")
    o2, l2 = ea.decode_paged(c.q.to(d), c.kv_pages.to(d), c.block_table.to(d), c.cache_seqlens.to(d), SCALE, dv=DV)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2.reshape(l1.shape))


def test_two_tokens_on_the_decode_workload_sampled():
    """Workload 5's lengths and cache with two query tokens per sequence;
    six sequences, both tokens, all heads, against the oracle."""
    cfg = inputs.DECODE_CONFIG
    gen = torch.Generator(device="cpu").manual_seed(int(cfg.seed))
    lens = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.B,), generator=gen, dtype=torch.int32)
    c = inputs.paged_decode_inputs(cfg.B, cfg.Hq, cfg.Dk, lens, cfg.page_size, cfg.seed + 200000, s_q=2)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    seqs = [0, 9, 21, 40, 55, 63]
    o_ref, lse_ref = _oracle(c, seqs=seqs)
    compare(o[seqs], lse[seqs], o_ref, lse_ref, "mtp decode workload 5, s_q=2 (sampled sequences)")


def test_maximum_query_units():
    """B * s_q = 2048 query units (512 sequences x 4 tokens), short sequences."""
    rng = np.random.default_rng(51)
    lens = rng.integers(0, 90, size=512).tolist()
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=51, s_q=4)
    o, lse = _run(c)
    assert ea.read_device_status(0) == 0
    seqs = [0, 100, 255, 511, int(np.argmax(lens))]
    o_ref, lse_ref = _oracle(c, seqs=seqs)
    compare(o[seqs], lse[seqs], o_ref, lse_ref, "mtp decode 2048 query units", o_max_abs=bf16_arith_bound(_vmax(c)))
