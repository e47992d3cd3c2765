"""Pins for the backward oracle (oracle.attention_bwd), CPU only.

The gradients are checked against things other than the function itself:
hand-derived cases (tests/golden/hand_worked_bwd.json), central finite differences of the forward oracle (the derivative by its
definition, no backward formula involved), torch autograd through fp64
scaled_dot_product_attention (independent library code), closed forms for a
single key and for the last key of a causal square problem, and the
translation invariance of softmax in the keys (the dK rows of a head sum to
zero).  The last test plants mistakes in copies of the oracle's source and
checks that the pins catch each one.
"""

import importlib
import inspect
import json
import math
import os
import textwrap

import numpy as np
import pytest
import torch

import oracle

# the package re-exports the function `attention`, which shadows the submodule name
oracle_attention = importlib.import_module("oracle.attention")


GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_bwd.json")


def _val(x):
    if isinstance(x, (int, float)):
        return float(x)
    sgn = -1.0 if x.startswith("-") else 1.0
    x = x.lstrip("-")
    if x == "ln3":
        return sgn * math.log(3.0)
    if x == "3ln3/4":
        return sgn * 3.0 * math.log(3.0) / 4.0
    raise ValueError(x)


def _arr(nested):
    return np.vectorize(_val, otypes=[np.float64])(np.array(nested, dtype=object))


with open(GOLDEN) as f:
    _G = json.load(f)["bwd"]


def _golden_check(fn, case):
    g = fn(_arr(case["q"]), _arr(case["k"]), _arr(case["v"]), _arr(case["do"]), case["causal"], case["scale"])
    for got, key in zip(g, ("dq", "dk", "dv")):
        np.testing.assert_allclose(got, _arr(case[key]), rtol=0, atol=1e-14, err_msg=f"{case['name']} {key}")


@pytest.mark.parametrize("case", _G, ids=[c["name"] for c in _G])
def test_hand_worked_cases(case):
    _golden_check(oracle.attention_bwd, case)


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _loss_grads_fd(q, k, v, do, causal, scale, h=1e-6):
    """Central differences of L = sum(dO * O) with O from the forward oracle."""

    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, causal, scale)
        return float(np.sum(o * do))

    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        it = np.nditer(args[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


FD_CASES = [
    # B, Nq, Nk, Hq, Hkv, D, Dv, causal
    (1, 3, 5, 2, 1, 3, 2, False),
    (1, 3, 5, 2, 1, 3, 3, True),
    (2, 4, 4, 2, 2, 2, 2, True),
    (1, 5, 3, 4, 2, 2, 3, True),   # Nq > Nk: the first two query rows see no key
]


def _fd_check(fn, case):
    B, Nq, Nk, Hq, Hkv, D, Dv, causal = case
    rng = np.random.default_rng(sum(case[:7]))
    q, k, v = _rand((B, Nq, Hq, D), rng), _rand((B, Nk, Hkv, D), rng), _rand((B, Nk, Hkv, Dv), rng)
    do = _rand((B, Nq, Hq, Dv), rng)
    dq, dk, dv = fn(q, k, v, do, causal, 0.8)
    fq, fk, fv = _loss_grads_fd(q, k, v, do, causal, 0.8)
    np.testing.assert_allclose(dq, fq, rtol=0, atol=1e-7)
    np.testing.assert_allclose(dk, fk, rtol=0, atol=1e-7)
    np.testing.assert_allclose(dv, fv, rtol=0, atol=1e-7)


@pytest.mark.parametrize("case", FD_CASES)
def test_matches_finite_differences(case):
    _fd_check(oracle.attention_bwd, case)


def _torch_check(fn, causal, Nq=37, Nk=45, Hq=4, Hkv=2, D=16, seed=7):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(2, Nq, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(2, Nk, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(2, Nk, Hkv, D, generator=g, dtype=torch.float64)
    do = torch.randn(2, Nq, Hq, D, generator=g, dtype=torch.float64)
    scale = 0.3
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    grp = Hq // Hkv
    kr = kt.repeat_interleave(grp, dim=2)
    vr = vt.repeat_interleave(grp, dim=2)
    mask = None
    if causal:
        mask = torch.arange(Nk)[None, :] <= torch.arange(Nq)[:, None] + (Nk - Nq)
    o = torch.nn.functional.scaled_dot_product_attention(qt.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2),
                                                         attn_mask=mask, scale=scale).transpose(1, 2)
    o.backward(do)
    dq, dk, dv = fn(q.numpy(), k.numpy(), v.numpy(), do.numpy(), causal, scale)
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=0, atol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_fp64(causal):
    _torch_check(oracle.attention_bwd, causal)


def _single_key_check(fn):
    """One key: every weight is 1, so dV = sum of dO over the group's query
    rows and heads, and the scores carry no gradient (dQ = dK = 0)."""
    rng = np.random.default_rng(3)
    q, k, v = _rand((2, 6, 4, 5), rng), _rand((2, 1, 2, 5), rng), _rand((2, 1, 2, 5), rng)
    do = _rand((2, 6, 4, 5), rng)
    dq, dk, dv = fn(q, k, v, do, False, 0.5)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    expect = do.reshape(2, 6, 2, 2, 5).sum(axis=(1, 3))
    np.testing.assert_allclose(dv[:, 0], expect, rtol=0, atol=1e-12)


def test_single_key_closed_form():
    _single_key_check(oracle.attention_bwd)


def _last_key_check(fn):
    """Causal with Nq = Nk: only the last query row sees the last key, so its
    dV is that row's weight on it times that row's dO."""
    rng = np.random.default_rng(11)
    N = 7
    q, k, v = _rand((1, N, 1, 4), rng), _rand((1, N, 1, 4), rng), _rand((1, N, 1, 4), rng)
    do = _rand((1, N, 1, 4), rng)
    scale = 0.6
    _, lse = oracle.attention(q, k, v, True, scale)
    p_last = np.exp(scale * q[0, N - 1, 0] @ k[0, N - 1, 0] - lse[0, 0, N - 1])
    _, _, dv = fn(q, k, v, do, True, scale)
    np.testing.assert_allclose(dv[0, N - 1, 0], p_last * do[0, N - 1, 0], rtol=0, atol=1e-12)


def test_causal_last_key_closed_form():
    _last_key_check(oracle.attention_bwd)


def _dk_sum_check(fn, causal):
    """Adding one vector to every key shifts each row of scores by a constant,
    which softmax ignores, so the dK rows of every KV head sum to zero."""
    rng = np.random.default_rng(5)
    q, k, v = _rand((2, 9, 4, 6), rng), _rand((2, 11, 2, 6), rng), _rand((2, 11, 2, 6), rng)
    do = _rand((2, 9, 4, 6), rng)
    _, dk, _ = fn(q, k, v, do, causal, 0.4)
    assert np.abs(dk.sum(axis=1)).max() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_dk_rows_sum_to_zero(causal):
    _dk_sum_check(oracle.attention_bwd, causal)


def test_row_and_head_subsets_match_full():
    rng = np.random.default_rng(8)
    q, k, v = _rand((1, 40, 4, 8), rng), _rand((1, 50, 2, 8), rng), _rand((1, 50, 2, 8), rng)
    do = _rand((1, 40, 4, 8), rng)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, True, 0.35, row_chunk=16)
    qr, kr = np.array([0, 7, 39]), np.array([1, 25, 49])
    sq, sk, sv = oracle.attention_bwd(q, k, v, do, True, 0.35, q_rows=qr, k_rows=kr, kv_heads=[1], row_chunk=7)
    np.testing.assert_allclose(sq[:, :, 2:], dq[:, qr, 2:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sk[:, :, 1], dk[:, kr, 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sv[:, :, 1], dv[:, kr, 1], rtol=0, atol=1e-12)
    assert not sq[:, :, :2].any() and not sk[:, :, 0].any()


def test_empty_inputs():
    q = np.zeros((1, 3, 2, 4))
    dq, dk, dv = oracle.attention_bwd(q, np.zeros((1, 0, 1, 4)), np.zeros((1, 0, 1, 4)), q, True, 0.5)
    assert dq.shape == (1, 3, 2, 4) and dk.shape == (1, 0, 1, 4) and not dq.any()


# ---------------------------------------------------------------- planted mistakes

_MUTATIONS = {
    "no_rowsum_term": ("dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))", "dS = P * dP"),
    "rowsum_sign": ("(dP - np.sum(P * dP", "(dP + np.sum(P * dP"),
    "dk_without_scale": ("dK[b, :, kv, :] += scale * (", "dK[b, :, kv, :] += 1.0 * ("),
    "dv_rows_shuffled": ("P[:, kr].T @ dOr", "P[:, kr].T @ dOr[::-1]"),
    "causal_off_by_one": ("rows[:, None] + (Nk - Nq)", "rows[:, None] + (Nk - Nq) - 1"),
    "dq_uses_v": ("scale * (dS[sel] @ Kmat)", "scale * (dS[sel] @ Vmat)"),
    "dk_uses_do": ("(dS[:, kr].T @ q[b, rows, hq, :])", "(dS[:, kr].T @ do[b, rows, hq, :])"),
}


def _mutant(name):
    old, new = _MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle_attention.attention_bwd))
    assert old in src, name
    ns = dict(vars(oracle_attention))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns["attention_bwd"]


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_pins_catch_planted_mistakes(name):
    fn = _mutant(name)
    checks = [lambda c=c: _fd_check(fn, c) for c in FD_CASES]
    checks += [lambda c=c: _torch_check(fn, c) for c in (False, True)]
    checks += [lambda: _single_key_check(fn), lambda: _last_key_check(fn)]
    checks += [lambda c=c: _golden_check(fn, c) for c in _G]
    checks += [lambda c=c: _dk_sum_check(fn, c) for c in (False, True)]
    failures = 0
    for chk in checks:
        try:
            chk()
        except (AssertionError, ValueError):   # a shape error is a caught mistake too
            failures += 1
    assert failures > 0, f"no pin caught the planted mistake {name}"
