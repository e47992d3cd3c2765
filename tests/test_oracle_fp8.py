"""Pins for the FP8 pieces of the oracle (oracle.e4m3_decode, oracle.attention_fp8), CPU only.

The E4M3 decoding is checked against torch's float8_e4m3fn (independent
library code) on all 256 codes and against values derived by hand from the
format's definition; attention_fp8 against a pure-Python brute force on the
decoded values.  Planted mistakes in copies of the decoder must fail a pin.
"""

import importlib
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch

import oracle

from exact_attention_135_b200 import inputs

oracle_attention = importlib.import_module("oracle.attention")

# (byte, value) derived from the definition: s eeee mmm, bias 7
HAND = [
    (0x00, 0.0), (0x80, -0.0),
    (0x38, 1.0),                      # e = 7, m = 0
    (0xB8, -1.0),
    (0x3C, 1.5),                      # e = 7, m = 4
    (0x40, 2.0),                      # e = 8
    (0x7E, 448.0),                    # e = 15, m = 6: 2^8 * 1.75, the largest finite value
    (0x77, 240.0),                    # e = 14, m = 7: 2^7 * 1.875
    (0x08, 2.0 ** -6),                # smallest normal
    (0x07, 7 * 2.0 ** -9),            # largest subnormal
    (0x01, 2.0 ** -9),                # smallest subnormal
    (0x81, -(2.0 ** -9)),
]


def _hand_check(fn):
    for code, val in HAND:
        got = float(fn(np.array([code], dtype=np.uint8))[0])
        assert got == val, (hex(code), got, val)
        assert math.copysign(1.0, got) == math.copysign(1.0, val), hex(code)
    nan = fn(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.all(np.isnan(nan))


def _torch_check(fn):
    codes = np.arange(256, dtype=np.uint8)
    ours = fn(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


def test_e4m3_hand_derived_codes():
    _hand_check(oracle.e4m3_decode)


def test_e4m3_matches_torch_on_every_code():
    _torch_check(oracle.e4m3_decode)


def test_quantized_inputs_decode_to_their_source_within_half_an_ulp():
    """The input recipe's bytes times the descale reproduce the fp32 draws to
    within e4m3 rounding (relative 2^-4 for normals, 2^-10 * descale absolute
    below the smallest normal)."""
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(4096, generator=gen)
    b, d = inputs.quantize_e4m3(x)
    back = d * oracle.e4m3_decode(b.numpy())
    xs = x.double().numpy()
    err = np.abs(back - xs)
    assert np.all(err <= np.maximum(np.abs(xs) * 2.0 ** -4, d * 2.0 ** -10) * (1 + 1e-12))
    assert abs(float(np.abs(back).max()) - float(np.abs(xs).max())) <= float(np.abs(xs).max()) * 2.0 ** -4
    assert np.float32(d) == d   # the descale is an fp32 value


def _brute(q, k, v, causal, scale):
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    g = Hq // Hkv
    O = np.zeros((B, Nq, Hq, D))
    for b in range(B):
        for h in range(Hq):
            for i in range(Nq):
                s = []
                for j in range(Nk):
                    if causal and j > i + Nk - Nq:
                        continue
                    s.append((scale * sum(q[b, i, h, d] * k[b, j, h // g, d] for d in range(D)), j))
                if not s:
                    continue
                m = max(x for x, _ in s)
                w = [(math.exp(x - m), j) for x, j in s]
                tot = sum(x for x, _ in w)
                for d in range(D):
                    O[b, i, h, d] = sum(x * v[b, j, h // g, d] for x, j in w) / tot
    return O


@pytest.mark.parametrize("causal", [False, True])
def test_attention_fp8_brute_force(causal):
    q8, k8, v8, (dq, dk, dv) = inputs.fp8_prefill_inputs(1, 4, 2, 3, 5, 4, seed=9)
    o, lse = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), dq, dk, dv, causal, 0.5)
    ref = _brute(dq * oracle.e4m3_decode(q8.numpy()), dk * oracle.e4m3_decode(k8.numpy()),
                 dv * oracle.e4m3_decode(v8.numpy()), causal, 0.5)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes

_MUTATIONS = {
    "bias_8": ("np.ldexp(1.0 + m / 8.0, e - 7)", "np.ldexp(1.0 + m / 8.0, e - 8)"),
    "subnormal_as_normal": ("np.where(e == 0, sub, normal)", "normal"),
    "sign_ignored": ("sign = np.where(c & 0x80, -1.0, 1.0)", "sign = 1.0"),
    "mantissa_over_16": ("m = (c & 0x7).astype(np.float64)", "m = (c & 0x7).astype(np.float64) / 2"),
    "no_nan": ("return np.where((e == 15) & (m == 7), np.nan, out)", "return out"),
}


def _mutant(name):
    old, new = _MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle_attention.e4m3_decode))
    assert old in src, name
    ns = dict(vars(oracle_attention))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns["e4m3_decode"]


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_pins_catch_planted_mistakes(name):
    fn = _mutant(name)
    failures = 0
    for chk in (lambda: _hand_check(fn), lambda: _torch_check(fn)):
        try:
            chk()
        except AssertionError:
            failures += 1
    assert failures == 2, f"a pin missed the planted mistake {name}"
