"""fp64 oracle of the KDA layer's input prologue (short convolution, Swish, L2Norm, gates).

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use it, and
it shares no code with the CUDA library.

Source: wiki page "Kimi Linear 高效注意力架构", section "模型架构": the KDA layer has
ShortConv + Swish activation + L2Norm (q/k), a low-rank channel-wise decay gate and a
sigmoid output gate + RMSNorm.  The page gives no formulas; the plainest reading,
per sequence (``cu_seqlens``), head h and channel c:

    conv(x)[t]  = sum_{w=0}^{W-1} weight[h, c, w] * x[t - w]      (x[t - w] = 0 before the
                                                                   sequence's first token)
    swish(z)    = z * sigmoid(z)
    q = l2norm(swish(conv_q(q_pre))),  k = l2norm(swish(conv_k(k_pre))),  v = swish(conv_v(v_pre))
    l2norm(z)   = z / sqrt(sum_c z_c^2 + eps)                     (over the head's d channels)
    log_alpha   = -rate[h] * softplus(a),   softplus(a) = log(1 + e^a)
    beta        = sigmoid(b)

``a`` is the low-rank gate's output (its projection is model-level) and ``rate`` a
positive per-head scale.  Parity status: pinned by ``tests/test_prologue_pins.py``.
"""
from __future__ import annotations

import numpy as np

from .epilogue import sigmoid


def softplus(x):
    """log(1 + e^x) in fp64 without overflow: max(x, 0) + log1p(e^{-|x|})."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def short_conv(x, weight, cu_seqlens):
    """Causal depthwise convolution over tokens, restarted at each sequence.

    x: [T, H, d]; weight: [H, d, W]; returns [T, H, d] in fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    weight = np.asarray(weight, dtype=np.float64)
    out = np.zeros_like(x)
    W = weight.shape[-1]
    for n in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[n]), int(cu_seqlens[n + 1])
        for t in range(s, e):
            for w in range(min(W, t - s + 1)):
                out[t] += weight[:, :, w] * x[t - w]
    return out


def swish(z):
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def l2norm(z, eps):
    z = np.asarray(z, dtype=np.float64)
    return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + float(eps))


def prologue(q_pre, k_pre, v_pre, w_q, w_k, w_v, a, rate, b, cu_seqlens, eps=1e-6):
    """The prologue's outputs (q, k, v, log_alpha, beta) in fp64 for packed sequences."""
    q = l2norm(swish(short_conv(q_pre, w_q, cu_seqlens)), eps)
    k = l2norm(swish(short_conv(k_pre, w_k, cu_seqlens)), eps)
    v = swish(short_conv(v_pre, w_v, cu_seqlens))
    log_alpha = -np.asarray(rate, np.float64)[None, :, None] * softplus(a)
    beta = sigmoid(b)
    return q, k, v, log_alpha, beta
