"""fp64 chunk-by-chunk (WY/UT) model of the KDA operator.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The wiki page "Kimi Linear 高效注意力架构", section "Kimi Delta Attention (KDA)",
says the operator has a hardware-efficient chunkwise form (its "硬件高效分块算法"
bullet) and gives its cost terms T d_k d_v + T C d_h + T C^2 (comparison table,
row "时间复杂度"); it does not print the chunk equations.  The rewrite below is
derived here from the state-update equation alone and is exact in real
arithmetic; ``tests/test_oracle_pins.py`` pins it to the token recurrence.

Within one chunk of L <= C tokens that starts from state S (rows r, i = tokens):

  g_r     = sum_{j <= r} log alpha_j          (inclusive, per key channel)
  u_r     = beta_r (v_r - S_{r-1}^T Diag(alpha_r) k_r)   so that
  S_r     = Diag(alpha_r) S_{r-1} + k_r u_r^T            (state-update equation)
  A_{ri}  = beta_r <k_r * exp(g_r - g_i), k_i>    for i < r, else 0
  T       = (I + A)^{-1} Diag(beta)                       (unit lower triangular)
  U       = T V - T (K * exp(g)) S                        (rows u_r)
  P_{ri}  = <q_r * exp(g_r - g_i), k_i>          for i <= r, else 0
  O       = (Q * exp(g)) S + P U                          (rows o_r = S_r^T q_r)
  S_next  = Diag(exp(g_L)) S + (K * exp(g_L - g))^T U

The decay between token i and a later token r, exp(g_r - g_i), is the product of the
alphas of tokens i+1 .. r.  The page's decay range alpha in [0, 1]^{d_k} (its
"Channel-wise 衰减" bullet) includes alpha = 0 (log alpha = -inf), where the running
sums g are -inf from that token on and g_r - g_i would be -inf - (-inf).  So every
exponent here is formed as a sum of log alpha over exactly the tokens it spans
(g_r - g_i over i+1 .. r, g_L - g_r over r+1 .. L), never as a difference of running
sums; nothing overflows and alpha = 0 gives exact zeros.  The chunk model is slow on
purpose and only runs on small inputs.
"""
from __future__ import annotations

import numpy as np


def chunk_stages(q, k, v, log_alpha, beta):
    """S-independent quantities of one chunk (fp64).

    q, k, log_alpha: [L, d_k]; v: [L, d_v]; beta: [L].
    Returns dict with g, A, T, P, Kg (= K*exp(g)), Qg (= Q*exp(g)),
    Khat (= K*exp(g_L - g)), Gamma (= exp(g_L)), Ut (= T V), W (= T Kg).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    b = np.asarray(beta, np.float64)
    L = q.shape[0]
    g = np.cumsum(la, axis=0)
    # decay between token i and a later token r, per channel: exp(sum of log alpha over
    # tokens i+1 .. r); zero for r < i (those pairs are masked out below)
    diff = np.zeros((L, L, la.shape[1]))                     # [r, i, d_k]
    for i in range(L):
        diff[i, i] = 1.0
        if i + 1 < L:
            diff[i + 1:, i] = np.exp(np.cumsum(la[i + 1:], axis=0))
    kk = np.einsum("rc,ic,ric->ri", k, k, diff)
    qk = np.einsum("rc,ic,ric->ri", q, k, diff)
    strict = np.tril(np.ones((L, L)), -1)
    incl = np.tril(np.ones((L, L)), 0)
    A = b[:, None] * kk * strict
    T = np.linalg.solve(np.eye(L) + A, np.diag(b))
    P = qk * incl
    Kg = k * np.exp(g)
    Qg = q * np.exp(g)
    # g_L - g_r = sum of log alpha over tokens r+1 .. L (zero for the last token)
    after = np.zeros_like(la)
    after[:-1] = np.cumsum(la[::-1], axis=0)[::-1][1:]
    Khat = k * np.exp(after)
    return dict(g=g, A=A, T=T, P=P, Kg=Kg, Qg=Qg, Khat=Khat, Gamma=np.exp(g[-1]),
                Ut=T @ v, W=T @ Kg)


def chunk_step(st, S):
    """Apply one chunk to state S [d_k, d_v]; return (O [L, d_v], S_next, U)."""
    U = st["Ut"] - st["W"] @ S
    O = st["Qg"] @ S + st["P"] @ U
    S_next = st["Gamma"][:, None] * S + st["Khat"].T @ U
    return O, S_next, U


def prefill(q, k, v, log_alpha, beta, cu_seqlens, S0=None, chunk: int = 64):
    """Chunked fp64 prefill over a packed batch; same shapes as ``oracle.prefill``.

    Chunks start at each sequence's first token and never cross a boundary; the
    last chunk of a sequence may be shorter than ``chunk``.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    b = np.asarray(beta, np.float64)
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = np.asarray(cu_seqlens, np.int64)
    N = cu.shape[0] - 1
    o = np.zeros((T, H, dv))
    S_out = np.zeros((N, H, dk, dv))
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[n, h], np.float64)
            for s in range(int(cu[n]), int(cu[n + 1]), chunk):
                e = min(s + chunk, int(cu[n + 1]))
                st = chunk_stages(q[s:e, h], k[s:e, h], v[s:e, h], la[s:e, h], b[s:e, h])
                O, S, _ = chunk_step(st, S)
                o[s:e, h] = O
            S_out[n, h] = S
    return o, S_out


def chunk_backward_unit(q, k, v, log_alpha, beta, dO, S0, dS_final, chunk: int = 64):
    """Gradients for one (sequence, head) unit by the chunk form, in fp64.

    The reverse of ``chunk_step`` taken product by product (the derivation is the chain
    rule through the chunk equations in this module's docstring), with the decay split
    at the chunk's middle token m as Kt = K e^{g - g_m}, Kb = K e^{g_m - g},
    Qt = Q e^{g - g_m} (so A = tril(Diag(beta) Kt Kb^T), P = tril_incl(Qt Kb^T)) and
    Kg = K e^{g}, Qg = Q e^{g}, Kh = K e^{g_L - g}.  q, k, log_alpha [L, d_k]; v, dO
    [L, d_v]; beta [L]; S0, dS_final [d_k, d_v].  Returns (dq, dk, dv, dlog_alpha, dbeta,
    dS0).  Pinned to the token adjoint in ``tests/test_backward_pins.py``.
    """
    q, k, v, la, b, dO = (np.asarray(x, np.float64) for x in (q, k, v, log_alpha, beta, dO))
    T, dk = q.shape
    starts = list(range(0, T, chunk))
    states = [np.array(S0, np.float64)]
    for s in starts[:-1] if starts else []:
        e = min(s + chunk, T)
        st = chunk_stages(q[s:e], k[s:e], v[s:e], la[s:e], b[s:e])
        states.append(chunk_step(st, states[-1])[1])
    dq, dkk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dla, db = np.zeros_like(la), np.zeros_like(b)
    dS = np.array(dS_final, np.float64)
    for ci in reversed(range(len(starts))):
        s = starts[ci]
        e = min(s + chunk, T)
        L = e - s
        S = states[ci]
        K, Q, V, B, dOc = k[s:e], q[s:e], v[s:e], b[s:e], dO[s:e]
        g = np.cumsum(la[s:e], axis=0)
        gm = g[(L - 1) // 2]
        gC = g[-1]
        Kt, Kb, Qt = K * np.exp(g - gm), K * np.exp(gm - g), Q * np.exp(g - gm)
        Kg, Qg, Kh = K * np.exp(g), Q * np.exp(g), K * np.exp(gC - g)
        strict, incl = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
        M = Kt @ Kb.T
        A = B[:, None] * M * strict
        X = np.linalg.inv(np.eye(L) + A)
        Tm = X * B[None, :]
        Pm = (Qt @ Kb.T) * incl
        Y = V - Kg @ S
        U = Tm @ Y
        # reverse of O = Qg S + Pm U and S_next = Diag(e^{g_C}) S + Kh^T U
        dU = Kh @ dS + Pm.T @ dOc
        dKh = U @ dS.T
        dQg = dOc @ S.T
        dP = (dOc @ U.T) * incl
        dQt = dP @ Kb
        dKb = dP.T @ Qt
        dT = dU @ Y.T
        dY = Tm.T @ dU
        dKg = -dY @ S.T
        dS_prev = np.exp(gC)[:, None] * dS + Qg.T @ dOc - Kg.T @ dY
        # T = X Diag(beta), X = (I + A)^{-1}, A = tril(Diag(beta) M)
        dbeta = np.sum(dT * X, axis=0)
        dA = -(X.T @ (dT * B[None, :]) @ X.T) * strict
        dbeta += np.sum(dA * M, axis=1)
        dM = B[:, None] * dA
        dKt = dM @ Kb
        dKb += dM.T @ Kt
        # back to q, k and the running sums g (g_m is a reference point: its gradient cancels)
        dq[s:e] = dQt * np.exp(g - gm) + dQg * np.exp(g)
        dkk[s:e] = dKt * np.exp(g - gm) + dKb * np.exp(gm - g) + dKg * np.exp(g) + dKh * np.exp(gC - g)
        dg = dKt * Kt - dKb * Kb + dQt * Qt + dKg * Kg + dQg * Qg - dKh * Kh
        dg[-1] += np.sum(dKh * Kh, axis=0) + np.exp(gC) * np.sum(dS * S, axis=1)
        dla[s:e] = np.cumsum(dg[::-1], axis=0)[::-1]
        dv[s:e] = dY
        db[s:e] = dbeta
        dS = dS_prev
    return dq, dkk, dv, dla, db, dS
