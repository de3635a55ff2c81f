"""fp64 oracle of the KDA layer's output epilogue: a sigmoid output gate with RMSNorm.

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use it, and
it shares no code with the CUDA library.

Source: wiki page "Kimi Linear 高效注意力架构", section "模型架构" (the KDA layer's
parts): the layer ends in a sigmoid output gate and an RMSNorm.  The page gives no
formula, so this takes the plainest reading, per head and token:

    y = o / sqrt(mean_j o_j^2 + eps)  (.)  w  (.)  sigmoid(gate),

with the mean over the d_v value channels of one head, a learned weight
w in R^{d_v} shared by the heads, eps added inside the square root, and the gate
pre-activation ``gate`` (same shape as o) produced elsewhere in the layer.

Parity status: pinned by ``tests/test_epilogue_pins.py`` (closed forms, invariants,
a hand-worked example and planted mistakes).
"""
from __future__ import annotations

import numpy as np


def sigmoid(x):
    """Logistic function 1 / (1 + e^{-x}) in fp64, written to avoid overflow."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def gated_rmsnorm(o, gate, weight, eps):
    """y = RMSNorm(o) * weight * sigmoid(gate) over the last axis (d_v), in fp64.

    o, gate: [..., d_v]; weight: [d_v]; eps >= 0.
    """
    o = np.asarray(o, dtype=np.float64)
    gate = np.asarray(gate, dtype=np.float64)
    weight = np.asarray(weight, dtype=np.float64)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + float(eps)) * weight * sigmoid(gate)
