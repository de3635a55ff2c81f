"""Pins of the input-prologue oracle (short conv, Swish, L2Norm, gates), independent of it.

Each pin is a fact the definitions fix; the planted mistakes at the end (each a
plausible slip) must fail at least one of them.
"""
import math

import numpy as np
import pytest

from oracle import prologue


def test_softplus_identities():
    x = np.linspace(-40, 40, 81)
    sp = prologue.softplus(x)
    assert np.allclose(sp - prologue.softplus(-x), x, atol=1e-12)  # softplus(x) - softplus(-x) = x
    assert abs(prologue.softplus(np.array([0.0]))[0] - math.log(2.0)) < 1e-15
    assert np.all(sp > 0) and np.all(np.isfinite(prologue.softplus(np.array([-1000.0, 1000.0]))))


def test_swish_values():
    # swish(0) = 0; swish(ln 3) = ln 3 * 3/4; swish(x) - swish(-x) = x
    assert prologue.swish(np.array([0.0]))[0] == 0.0
    assert abs(prologue.swish(np.array([math.log(3.0)]))[0] - 0.75 * math.log(3.0)) < 1e-15
    x = np.linspace(-20, 20, 41)
    assert np.allclose(prologue.swish(x) - prologue.swish(-x), x, atol=1e-12)


def test_conv_delta_kernels_shift_within_sequences():
    # a weight of 1 at tap w delays the input by w tokens, zero-filled at each sequence start
    rng = np.random.default_rng(1)
    cu = [0, 5, 5, 12]
    x = rng.standard_normal((12, 2, 3))
    for w in range(4):
        wt = np.zeros((2, 3, 4))
        wt[:, :, w] = 1.0
        y = prologue.short_conv(x, wt, cu)
        for s, e in [(0, 5), (5, 12)]:
            for t in range(s, e):
                expect = x[t - w] if t - w >= s else np.zeros((2, 3))
                assert np.array_equal(y[t], expect)


def test_conv_hand_worked_and_per_channel():
    # one sequence, x = (1, 2, 3, 4), weight (0.5, 0.25, 1.0): y = (0.5, 1.25, 3, 4.75)
    x = np.array([1.0, 2.0, 3.0, 4.0]).reshape(4, 1, 1)
    y = prologue.short_conv(x, np.array([0.5, 0.25, 1.0]).reshape(1, 1, 3), [0, 4])
    assert np.allclose(y.ravel(), [0.5, 1.25, 3.0, 4.75])
    # channels and heads use their own weights only
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 2, 3))
    wt = rng.standard_normal((2, 3, 4))
    y = prologue.short_conv(x, wt, [0, 6])
    t, h, c = 5, 1, 2
    assert abs(y[t, h, c] - sum(wt[h, c, w] * x[t - w, h, c] for w in range(4))) < 1e-13


def test_l2norm_unit_rows_and_eps():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((7, 2, 16))
    n = prologue.l2norm(z, 0.0)
    assert np.allclose(np.sum(n * n, -1), 1.0, rtol=1e-13)
    # hand-worked: (3, 4) with eps = 11 -> (3, 4) / 6
    assert np.allclose(prologue.l2norm(np.array([[3.0, 4.0]]), 11.0), [[0.5, 4.0 / 6.0]])


def test_gates_closed_forms_and_end_to_end():
    rng = np.random.default_rng(4)
    T, H, d = 9, 2, 4
    qp, kp, vp = (rng.standard_normal((T, H, d)) for _ in range(3))
    ident = np.zeros((H, d, 4))
    ident[:, :, 0] = 1.0
    a = rng.standard_normal((T, H, d))
    b = rng.standard_normal((T, H))
    rate = np.array([0.1, 2.0])
    q, k, v, la, beta = prologue.prologue(qp, kp, vp, ident, ident, ident, a, rate, b, [0, T], eps=0.0)
    sw = lambda z: z / (1.0 + np.exp(-z))
    assert np.allclose(v, sw(vp), rtol=1e-13)
    assert np.allclose(q, sw(qp) / np.linalg.norm(sw(qp), axis=-1, keepdims=True), rtol=1e-12)
    assert np.allclose(la[:, 1], -2.0 * np.log1p(np.exp(a[:, 1])), rtol=1e-13)
    assert np.all(la <= 0) and np.allclose(beta, 1.0 / (1.0 + np.exp(-b)), rtol=1e-14)
    # log alpha = 0 exactly needs a -> -inf; a = 0 gives -rate ln 2
    la0 = prologue.prologue(qp, kp, vp, ident, ident, ident, np.zeros_like(a), rate, b, [0, T])[3]
    assert np.allclose(la0[:, 0], -0.1 * math.log(2.0), rtol=1e-14)


def _mutants():
    P = prologue
    conv = prologue.short_conv  # the original, captured before any patching

    def conv_leaks(x, weight, cu):  # ignores sequence starts
        return conv(x, weight, [0, len(x)])

    def conv_anticausal(x, weight, cu):
        return np.ascontiguousarray(conv(np.asarray(x)[::-1], weight, [0, len(x)])[::-1])

    def swish_is_silu_squared(z):
        return z * P.sigmoid(z) ** 2

    def l2_mean(z, eps):
        return z / np.sqrt(np.mean(z * z, axis=-1, keepdims=True) + eps)

    def softplus_no_log(x):
        return np.maximum(np.asarray(x, np.float64), 0.0) + np.exp(-np.abs(x))

    return [("short_conv", conv_leaks), ("short_conv", conv_anticausal), ("swish", swish_is_silu_squared),
            ("l2norm", l2_mean), ("softplus", softplus_no_log)]


@pytest.mark.parametrize("name,mutant", _mutants(), ids=lambda x: x if isinstance(x, str) else x.__name__)
def test_planted_mistakes_fail_a_pin(name, mutant, monkeypatch):
    monkeypatch.setattr(prologue, name, mutant)
    pins = [test_softplus_identities, test_swish_values, test_conv_delta_kernels_shift_within_sequences,
            test_conv_hand_worked_and_per_channel, test_l2norm_unit_rows_and_eps,
            test_gates_closed_forms_and_end_to_end]
    failed = 0
    for p in pins:
        try:
            p()
        except AssertionError:
            failed += 1
    assert failed >= 1, f"{mutant.__name__} passed every pin"
