"""GPU test of attn_decode_paged_noalloc, the decode entry point for callers
that cannot allocate device memory at decode time (for example a serving
engine that gives all of HBM to its KV-cache pool, or a latency-critical loop
that may not call the allocator).  Its split-KV scratch is a fixed array
inside the library instead of a caller workspace.

The test calls it through the C ABI twice in a row and checks each result
against the workspace-taking entry point on the same inputs.  This file is
collected last, so a run that stops at the first failure has already run
every other test; it also passes when run alone in a fresh process.
"""

import math

import pytest
import torch

import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import O_MAX_ABS, O_REL_RMS, LSE_MAX_ABS

pytestmark = pytest.mark.gpu

HQ, DK, DV, PAGE = 128, 576, 512, 64


def _close(o_a, l_a, o_b, l_b):
    d = (o_a.float() - o_b.float())
    assert d.abs().max().item() <= O_MAX_ABS
    assert (d.norm() / o_b.float().norm()).item() <= O_REL_RMS
    fin = torch.isfinite(l_b)
    assert torch.equal(torch.isneginf(l_a), torch.isneginf(l_b))
    assert (l_a[fin] - l_b[fin]).abs().max().item() <= LSE_MAX_ABS


def test_noalloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda:0")
    lens = [1500, 0, 64, 8000, 333, 4097]
    c = inputs.paged_decode_inputs(len(lens), HQ, DK, lens, PAGE, seed=4242)
    q, kv, bt, sl = c.q.to(dev), c.kv_pages.to(dev), c.block_table.to(dev), c.cache_seqlens.to(dev)
    scale = 1.0 / math.sqrt(192.0)
    lib = ea.library()
    assert lib.attn_decode_paged_noalloc_max_bytes() >= ea.decode_workspace_size(len(lens), HQ, DV)

    o_ref, l_ref = ea.decode_paged(q, kv, bt, sl, scale, dv=DV)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full((len(lens), 1, HQ, DV), 7.0, dtype=torch.bfloat16, device=dev)
        lse = torch.full((len(lens), HQ), 7.0, dtype=torch.float32, device=dev)
        rc = lib.attn_decode_paged_noalloc(q.data_ptr(), kv.data_ptr(), bt.data_ptr(), sl.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), len(lens), HQ, DK, DV, PAGE,
                                           kv.shape[0], bt.shape[1], scale,
                                           torch.cuda.current_stream(dev).cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert ea.read_device_status(0) == 0
        _close(o, lse, o_ref, l_ref)


def test_noalloc_rejects_batches_beyond_the_batch_limit():
    lib = ea.library()
    # B above the decode's batch limit (2048 sequences): rejected on the host,
    # nothing enqueued.  The array-size check itself is not reached on a
    # 148-SM B200: the largest workspace (2048 sequences) fits in the array.
    A = 0x10000
    rc = lib.attn_decode_paged_noalloc(A, A, A, A, A, A, 5000, HQ, DK, DV, PAGE, 10, 10, 0.1, None)
    assert rc == 2
    assert ea.decode_workspace_size(2048, HQ, DV, 0) <= lib.attn_decode_paged_noalloc_max_bytes()
