"""Failure detection without a GPU fault.

A kernel waits on a barrier that nothing releases, with the library's own
bounded wait (limit 50 ms).  The wait gives up, the device status word reads
ATTN_ERR_TIMEOUT, and the context keeps working: an attention call right
after it is still exact.  Nothing traps, faults or hangs.
"""

import math

import pytest
import torch

import oracle
import exact_attention_135_b200 as ea
from exact_attention_135_b200 import inputs
from parity import compare, to_np64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    dev = torch.device("cuda:0")
    lib = ea.library()
    assert ea.read_device_status(0) == 0
    rc = lib.attn_selftest_wait_timeout(50_000, torch.cuda.current_stream(dev).cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert ea.read_device_status(0) == 4          # ATTN_ERR_TIMEOUT
    assert ea.read_device_status(0) == 0          # cleared by the read
    # the context is still usable and exact
    q, k, v = inputs.prefill_inputs(1, 2, 2, 200, 200, 64, 64, seed=21)
    o, lse = ea.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True, scale=1 / math.sqrt(64))
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention(to_np64(q), to_np64(k), to_np64(v), True, 1 / math.sqrt(64))
    compare(o, lse, o_ref, lse_ref, "after timeout self-test")
    assert ea.read_device_status(0) == 0


def test_selftest_rejects_bad_limits():
    lib = ea.library()
    assert lib.attn_selftest_wait_timeout(0, None) == 1
    assert lib.attn_selftest_wait_timeout(20_000_000, None) == 1
