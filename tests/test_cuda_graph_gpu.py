"""CUDA-graph capture and replay of the C-ABI entry points.

Every entry point only enqueues work on the caller's stream, and the decodes
plan their split on the device from cache_seqlens (the split kernel builds
the prefix sums itself).  So one graph captured with caller-owned outputs and
workspace serves later steps whose inputs are rewritten in place, sequence
lengths included, with no host planning between replays.  A replay must give
exactly what an eager call on the same inputs gives, bit for bit (except the
backward's dQ, whose fp32 adds land in arrival order), and the replays are
checked against the fp64 oracle as the other parity tests are.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import compare, to_np64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
PAGE = 64


def _capture(fn):
    """Run fn once on a side stream (first-call set-up stays out of the
    capture), then capture it into a graph."""
    side = torch.cuda.Stream(device=DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(DEV).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 0
    return g


def _bf16(shape, seed):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=gen).to(torch.bfloat16)


def test_mla_decode_graph_follows_new_queries_and_lengths():
    HQ, DK, DV = 128, 576, 512
    scale = 1.0 / math.sqrt(192.0)
    lens1 = [100, 2000, 64, 0, 5000, 333, 1, 4096]
    # every length at most the first step's, so the block table still covers it
    lens2 = [99, 1, 64, 0, 4097, 333, 0, 2500]
    c = inputs.paged_decode_inputs(len(lens1), HQ, DK, lens1, PAGE, seed=71)
    B = len(lens1)
    q, kv, bt, sl = (t.to(DEV) for t in (c.q, c.kv_pages, c.block_table, c.cache_seqlens))
    o = torch.empty((B, 1, HQ, DV), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, HQ), dtype=torch.float32, device=DEV)
    ws = torch.empty(max(ea.decode_workspace_size(B, HQ, DV, DEV), 1), dtype=torch.uint8, device=DEV)
    g = _capture(lambda: ea.decode_paged(q, kv, bt, sl, scale, dv=DV, out=o, lse=lse, workspace=ws))

    pages = to_np64(c.kv_pages)[:, :, 0]
    for step, (q_host, lens) in enumerate(((_bf16(c.q.shape, 72), lens2), (c.q, lens1))):
        q.copy_(q_host.to(DEV))
        sl.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        o_e, lse_e = ea.decode_paged(q, kv, bt, sl, scale, dv=DV)
        torch.cuda.synchronize()
        assert ea.read_device_status(0) == 0
        assert torch.equal(o, o_e), step
        assert torch.equal(lse, lse_e), step
        o_ref, lse_ref = oracle.decode_paged(to_np64(q_host)[:, 0], pages, c.block_table.numpy(),
                                             np.asarray(lens, dtype=np.int32), scale, DV, page_size=PAGE)
        compare(o[:, 0], lse, o_ref, lse_ref, f"MLA decode graph replay {step}, lens={lens}")


def test_gqa_decode_graph_follows_new_queries_and_lengths():
    HQ, HKV, D = 32, 8, 128
    scale = 1.0 / math.sqrt(D)
    lens1 = [700, 0, 3000, 64, 1, 1500]
    lens2 = [650, 0, 65, 64, 1, 1499]
    c = inputs.paged_gqa_decode_inputs(len(lens1), HQ, HKV, D, lens1, PAGE, seed=81)
    B = len(lens1)
    q, kp, vp, bt, sl = (t.to(DEV) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.cache_seqlens))
    o = torch.empty((B, 1, HQ, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, HQ), dtype=torch.float32, device=DEV)
    ws = torch.empty(max(ea.decode_gqa_workspace_size(B, HQ, HKV, D, DEV), 1), dtype=torch.uint8, device=DEV)
    g = _capture(lambda: ea.decode_paged_gqa(q, kp, vp, bt, sl, scale, out=o, lse=lse, workspace=ws))

    k64, v64 = to_np64(c.k_pages), to_np64(c.v_pages)
    for step, (q_host, lens) in enumerate(((_bf16(c.q.shape, 82), lens2), (c.q, lens1))):
        q.copy_(q_host.to(DEV))
        sl.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        o_e, lse_e = ea.decode_paged_gqa(q, kp, vp, bt, sl, scale)
        torch.cuda.synchronize()
        assert ea.read_device_status(0) == 0
        assert torch.equal(o, o_e), step
        assert torch.equal(lse, lse_e), step
        o_ref, lse_ref = oracle.decode_paged_gqa(to_np64(q_host)[:, 0], k64, v64, c.block_table.numpy(),
                                                 np.asarray(lens, dtype=np.int32), scale, page_size=PAGE)
        compare(o[:, 0], lse, o_ref, lse_ref, f"GQA decode graph replay {step}, lens={lens}")


@pytest.mark.parametrize("D", [64, 128])
def test_training_step_graph_replay(D):
    """Forward and backward captured together, replayed on new Q, K, V, dO."""
    B, HQ, HKV, N = 1, 4, 2, 300
    scale = 1.0 / math.sqrt(D)
    host = [inputs.bwd_inputs(B, HQ, HKV, N, N, D, seed) for seed in (91, 92)]
    q, k, v, do = (t.to(DEV) for t in host[0])
    o = torch.empty((B, N, HQ, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, HQ, N), dtype=torch.float32, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(ea.bwd_workspace_size(B, HQ, N, D), 1), dtype=torch.uint8, device=DEV)

    def step():
        ea.fwd(q, k, v, causal=True, scale=scale, out=o, lse=lse)
        ea.bwd(q, k, v, o, lse, do, causal=True, scale=scale, dq=dq, dk=dk, dv=dv, workspace=ws)

    g = _capture(step)
    for i in (1, 0):
        for dst, src in zip((q, k, v, do), host[i]):
            dst.copy_(src.to(DEV))
        g.replay()
        o_e, lse_e = ea.fwd(q, k, v, causal=True, scale=scale)
        dq_e, dk_e, dv_e = ea.bwd(q, k, v, o_e, lse_e, do, causal=True, scale=scale)
        torch.cuda.synchronize()
        assert ea.read_device_status(0) == 0
        assert torch.equal(o, o_e) and torch.equal(lse, lse_e), i
        assert torch.equal(dk, dk_e) and torch.equal(dv, dv_e), i
        # dQ: the same fp32 terms added in another order, then rounded to bf16
        assert float((dq.float() - dq_e.float()).abs().max()) <= 2.0 ** -7 * float(dq_e.float().abs().max()), i
        o_ref, lse_ref = oracle.attention(*(to_np64(t) for t in host[i][:3]), True, scale)
        compare(o, lse, o_ref, lse_ref, f"training-step graph replay, D={D}, inputs {i}")
