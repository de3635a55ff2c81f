"""Pins of the output-epilogue oracle (sigmoid gate + RMSNorm), independent of it.

Each pin is a fact of the arithmetic the epilogue's definition fixes, chosen so a
plausible mistake (sum for mean, eps outside the root, a missing weight, the mean
over the wrong axis, another gate function) fails at least one of them; the
planted mistakes at the end check exactly that.
"""
import math

import numpy as np
import pytest

from oracle import epilogue


def test_sigmoid_values():
    # sigma(0) = 1/2; sigma(ln 3) = 1 / (1 + 1/3) = 3/4; sigma(-x) = 1 - sigma(x)
    assert epilogue.sigmoid(np.array([0.0]))[0] == 0.5
    assert abs(epilogue.sigmoid(np.array([math.log(3.0)]))[0] - 0.75) < 1e-15
    x = np.linspace(-30, 30, 61)
    assert np.allclose(epilogue.sigmoid(-x), 1.0 - epilogue.sigmoid(x), atol=1e-15)
    assert np.all(np.isfinite(epilogue.sigmoid(np.array([-800.0, 800.0]))))


def test_hand_worked_example():
    # o = (3, 4): mean square 12.5; eps = 0.5 -> root 13; w = (1, 2); gate = (0, ln 3)
    # y = (3 / sqrt 13 * 1 * 1/2, 4 / sqrt 13 * 2 * 3/4) = (1.5, 6) / sqrt 13
    y = epilogue.gated_rmsnorm(np.array([[3.0, 4.0]]), np.array([[0.0, math.log(3.0)]]),
                               np.array([1.0, 2.0]), 0.5)
    assert np.allclose(y, np.array([[1.5, 6.0]]) / math.sqrt(13.0), rtol=1e-14)


def test_constant_vector_closed_form():
    # o = c 1 with eps = 0: the RMS is |c|, so y = sign(c) w sigma(g)
    rng = np.random.default_rng(1)
    dv = 8
    w = rng.standard_normal(dv)
    g = rng.standard_normal((2, dv))
    o = np.stack([np.full(dv, 2.5), np.full(dv, -0.25)])
    y = epilogue.gated_rmsnorm(o, g, w, 0.0)
    assert np.allclose(y[0], w * epilogue.sigmoid(g[0]), rtol=1e-14)
    assert np.allclose(y[1], -w * epilogue.sigmoid(g[1]), rtol=1e-14)


def test_unit_rms_and_scale_invariance():
    # with w = 1, a saturated gate and eps = 0 the output has mean square 1 per row,
    # and scaling o by lambda > 0 leaves y unchanged; negating o negates y
    rng = np.random.default_rng(2)
    o = rng.standard_normal((5, 3, 16))
    big = np.full(o.shape, 60.0)
    y = epilogue.gated_rmsnorm(o, big, np.ones(16), 0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-13)
    g = rng.standard_normal(o.shape)
    w = rng.standard_normal(16)
    y1 = epilogue.gated_rmsnorm(o, g, w, 0.0)
    assert np.allclose(epilogue.gated_rmsnorm(7.5 * o, g, w, 0.0), y1, rtol=1e-13)
    assert np.allclose(epilogue.gated_rmsnorm(-o, g, w, 0.0), -y1, rtol=1e-13)


def test_rows_are_independent():
    # every (token, head) row is normalised on its own: changing one row changes no other
    rng = np.random.default_rng(3)
    o = rng.standard_normal((4, 2, 8))
    g = rng.standard_normal(o.shape)
    w = rng.standard_normal(8)
    y = epilogue.gated_rmsnorm(o, g, w, 1e-6)
    o2 = o.copy()
    o2[1, 0] *= 100.0
    y2 = epilogue.gated_rmsnorm(o2, g, w, 1e-6)
    mask = np.ones((4, 2), bool)
    mask[1, 0] = False
    assert np.array_equal(y[mask], y2[mask])


def test_eps_inside_the_root():
    # o = 0 gives y = 0 for eps > 0; a tiny row is damped by eps: y = o / sqrt(ms + eps)
    y0 = epilogue.gated_rmsnorm(np.zeros((1, 4)), np.zeros((1, 4)), np.ones(4), 1e-6)
    assert np.array_equal(y0, np.zeros((1, 4)))
    o = np.full((1, 4), 1e-3)  # ms = 1e-6
    y = epilogue.gated_rmsnorm(o, np.full((1, 4), 60.0), np.ones(4), 3e-6)
    assert np.allclose(y, 1e-3 / math.sqrt(4e-6), rtol=1e-13)


def _mutants():
    s = epilogue.sigmoid

    def sum_not_mean(o, g, w, eps):
        return o / np.sqrt(np.sum(o * o, -1, keepdims=True) + eps) * w * s(g)

    def eps_outside(o, g, w, eps):
        return o / (np.sqrt(np.mean(o * o, -1, keepdims=True)) + eps) * w * s(g)

    def no_weight(o, g, w, eps):
        return o / np.sqrt(np.mean(o * o, -1, keepdims=True) + eps) * s(g)

    def wrong_axis(o, g, w, eps):
        return o / np.sqrt(np.mean(o * o, 0, keepdims=True) + eps) * w * s(g)

    def silu_gate(o, g, w, eps):
        return o / np.sqrt(np.mean(o * o, -1, keepdims=True) + eps) * w * (g * s(g))

    def gate_before_norm(o, g, w, eps):
        og = o * s(g)
        return og / np.sqrt(np.mean(og * og, -1, keepdims=True) + eps) * w

    return [sum_not_mean, eps_outside, no_weight, wrong_axis, silu_gate, gate_before_norm]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_planted_mistakes_fail_a_pin(mutant, monkeypatch):
    monkeypatch.setattr(epilogue, "gated_rmsnorm", mutant)
    pins = [test_hand_worked_example, test_constant_vector_closed_form,
            test_unit_rms_and_scale_invariance, test_rows_are_independent, test_eps_inside_the_root]
    failed = 0
    for p in pins:
        try:
            p()
        except AssertionError:
            failed += 1
    assert failed >= 1, f"{mutant.__name__} passed every pin"
