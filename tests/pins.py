"""Pins for the fp64 KDA oracle: checks fixed by the pages and by mathematics.

Each ``pin_*`` takes ``run(q, k, v, log_alpha, beta, cu_seqlens, S0) -> (o, S)``
(the oracle's prefill signature, fp64 numpy in and out) and raises
AssertionError when the oracle disagrees with the fixed fact.  The same pins
run against deliberately broken copies of the oracle in
``test_oracle_mutants.py``: every planted mistake must fail at least one.

Sources: the wiki page "Kimi Linear 高效注意力架构", section "Kimi Delta
Attention (KDA)" (state-update equation; channel-wise decay alpha in
[0,1]^{d_k}; rank-1 Householder-like delta-rule correction), its section
"线性注意力演进" (linear attention = no decay and an unbounded sum; DeltaNet =
delta rule; Gated DeltaNet = delta rule with a head-wise scalar gate), and the
delta-rule read-out o_t = S_t^T q_t of the post-update state.
"""
from __future__ import annotations

import json
import os

import numpy as np

RTOL = 1e-12
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_err(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return num / den if den > 0 else num


def _rand_case(rng, T, H, dk, dv, unit_k=True):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -0.3 * np.log1p(np.exp(rng.standard_normal((T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, la, b


def _single(T):
    return np.array([0, T], np.int64)


def pin_hand_worked(run):
    """The three-token d=2 example worked by hand (tests/golden/hand_worked_d2.json)."""
    with open(os.path.join(GOLDEN, "hand_worked_d2.json")) as f:
        ex = json.load(f)
    toks = ex["tokens"]
    T = len(toks)
    q = np.array([t["q"] for t in toks], np.float64)[:, None, :]
    k = np.array([t["k"] for t in toks], np.float64)[:, None, :]
    v = np.array([t["v"] for t in toks], np.float64)[:, None, :]
    la = np.log(np.array([t["alpha"] for t in toks], np.float64))[:, None, :]
    b = np.array([t["beta"] for t in toks], np.float64)[:, None]
    S0 = np.array(ex["S0"], np.float64)[None, None]
    o, S = run(q, k, v, la, b, _single(T), S0)
    exp_o = np.array([t["o"] for t in toks])
    np.testing.assert_allclose(o[:, 0, :], exp_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], np.array(toks[-1]["S"]), rtol=0, atol=1e-12)
    # every prefix of the sequence ends in the printed intermediate state
    for t in range(1, T):
        _, St = run(q[:t], k[:t], v[:t], la[:t], b[:t], _single(t), S0)
        np.testing.assert_allclose(St[0, 0], np.array(toks[t - 1]["S"]), rtol=0, atol=1e-12)


def pin_beta_zero_closed_form(run, seed=1):
    """beta == 0 removes erase and write: S_t = Diag(exp(sum_{s<=t} log alpha_s)) S0."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 9, 2, 5, 3
    q, k, v, la, _ = _rand_case(rng, T, H, dk, dv)
    b = np.zeros((T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = run(q, k, v, la, b, _single(T), S0)
    G = np.cumsum(la, axis=0)                        # [T, H, dk]
    for h in range(H):
        for t in range(T):
            St = np.exp(G[t, h])[:, None] * S0[0, h]
            assert rel_err(o[t, h], St.T @ q[t, h]) < RTOL
        assert rel_err(S[0, h], np.exp(G[-1, h])[:, None] * S0[0, h]) < RTOL


def pin_exact_reconstruction(run, seed=2):
    """beta = 1 and ||k_t|| = 1: the delta rule stores v_t exactly, k_t^T S_t = v_t^T,
    for any decay and any earlier state (every prefix is checked)."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 7, 2, 6, 4
    q, k, v, la, _ = _rand_case(rng, T, H, dk, dv, unit_k=True)
    b = np.ones((T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    for t in range(1, T + 1):
        _, St = run(q[:t], k[:t], v[:t], la[:t], b[:t], _single(t), S0)
        for h in range(H):
            np.testing.assert_allclose(k[t - 1, h] @ St[0, h], v[t - 1, h], rtol=0, atol=1e-12)


def pin_orthonormal_linear_attention(run, seed=3):
    """alpha == 1, beta == 1, mutually orthonormal keys, S0 = 0: every erase hits an
    empty direction, so the state is the linear-attention sum S_T = K^T V and
    o_t = sum_{i<=t} (q_t . k_i) v_i (causal linear attention)."""
    rng = np.random.default_rng(seed)
    dk, dv, T, H = 8, 5, 6, 1
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:T][:, None, :]                            # T orthonormal rows
    q = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    la = np.zeros((T, H, dk))
    b = np.ones((T, H))
    o, S = run(q, k, v, la, b, _single(T), None)
    K, V = k[:, 0], v[:, 0]
    assert rel_err(S[0, 0], K.T @ V) < RTOL
    ref_o = np.stack([sum((q[t, 0] @ K[i]) * V[i] for i in range(t + 1)) for t in range(T)])
    assert rel_err(o[:, 0], ref_o) < RTOL


def pin_scalar_gate_gdn(run, seed=4, ungated=False):
    """alpha_t = a_t * 1 (one gate per head) gives Gated DeltaNet, written here as
    S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T with explicit
    matrices; ungated=True (a_t = 1) gives DeltaNet."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 8, 2, 4, 6
    q, k, v, _, b = _rand_case(rng, T, H, dk, dv, unit_k=False)
    a = np.ones((T, H)) if ungated else rng.uniform(0.3, 1.0, (T, H))
    la = np.repeat(np.log(a)[:, :, None], dk, axis=2)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = run(q, k, v, la, b, _single(T), S0)
    for h in range(H):
        St = S0[0, h].copy()
        for t in range(T):
            kt = k[t, h][:, None]
            St = a[t, h] * (np.eye(dk) - b[t, h] * kt @ kt.T) @ St + b[t, h] * kt @ v[t, h][None]
            assert rel_err(o[t, h], St.T @ q[t, h]) < RTOL
        assert rel_err(S[0, h], St) < RTOL


def pin_bruteforce_products(run, seed=5):
    """Tiny inputs: M_t = (I - beta_t k_t k_t^T) Diag(alpha_t) as explicit matrices;
    S_t = M_t ... M_1 S0 + sum_{s<=t} M_t ... M_{s+1} beta_s k_s v_s^T."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 6, 1, 4, 3
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv, unit_k=False)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = run(q, k, v, la, b, _single(T), S0)
    M = [(np.eye(dk) - b[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(la[t, 0]))
         for t in range(T)]

    def prod(hi, lo):  # M_hi ... M_lo (identity when hi < lo)
        R = np.eye(dk)
        for s in range(lo, hi + 1):
            R = M[s] @ R
        return R

    for t in range(T):
        St = prod(t, 0) @ S0[0, 0]
        for s in range(t + 1):
            St = St + prod(t, s + 1) @ (b[s, 0] * np.outer(k[s, 0], v[s, 0]))
        assert rel_err(o[t, 0], St.T @ q[t, 0]) < RTOL
    assert rel_err(S[0, 0], St) < RTOL


def pin_scalar_d1(run, seed=6):
    """d_k = d_v = 1: s_t = (1 - beta_t k_t^2) alpha_t s_{t-1} + beta_t k_t v_t, o_t = q_t s_t."""
    rng = np.random.default_rng(seed)
    T = 12
    q, k, v = (rng.standard_normal((T, 1, 1)) for _ in range(3))
    la = -rng.uniform(0, 1, (T, 1, 1))
    b = rng.uniform(0, 1, (T, 1))
    o, S = run(q, k, v, la, b, _single(T), np.array([[[[0.7]]]]))
    s = 0.7
    for t in range(T):
        s = (1 - b[t, 0] * k[t, 0, 0] ** 2) * np.exp(la[t, 0, 0]) * s + b[t, 0] * k[t, 0, 0] * v[t, 0, 0]
        assert abs(o[t, 0, 0] - q[t, 0, 0] * s) < 1e-12 * max(1.0, abs(q[t, 0, 0] * s))
    assert abs(S[0, 0, 0, 0] - s) < 1e-12 * max(1.0, abs(s))


def pin_linearity(run, seed=7):
    """For fixed q, k, alpha, beta the map (S0, V) -> (o, S_T) is linear."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 10, 2, 5, 4
    q, k, v1, la, b = _rand_case(rng, T, H, dk, dv)
    v2 = rng.standard_normal(v1.shape)
    A1 = rng.standard_normal((1, H, dk, dv))
    A2 = rng.standard_normal((1, H, dk, dv))
    c1, c2 = 0.7, -1.3
    cu = _single(T)
    o1, S1 = run(q, k, v1, la, b, cu, A1)
    o2, S2 = run(q, k, v2, la, b, cu, A2)
    o3, S3 = run(q, k, c1 * v1 + c2 * v2, la, b, cu, c1 * A1 + c2 * A2)
    assert rel_err(o3, c1 * o1 + c2 * o2) < 1e-11
    assert rel_err(S3, c1 * S1 + c2 * S2) < 1e-11


def pin_householder_norms(run, seed=8):
    """v = 0: with beta = 2, ||k|| = 1, alpha = 1 every step is the reflection
    I - 2 k k^T, so ||S||_F is preserved; with beta in [0,1] and alpha in (0,1]
    every step is a contraction, so ||S||_2 never grows."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 8, 1, 5, 3
    q, k, _, la, b = _rand_case(rng, T, H, dk, dv, unit_k=True)
    v = np.zeros((T, H, dv))
    S0 = rng.standard_normal((1, H, dk, dv))
    _, S = run(q, k, v, np.zeros_like(la), 2.0 * np.ones((T, H)), _single(T), S0)
    assert abs(np.linalg.norm(S[0, 0]) - np.linalg.norm(S0[0, 0])) < 1e-12 * np.linalg.norm(S0[0, 0])
    prev = np.linalg.norm(S0[0, 0], 2)
    for t in range(1, T + 1):
        _, St = run(q[:t], k[:t], v[:t], la[:t], b[:t], _single(t), S0)
        cur = np.linalg.norm(St[0, 0], 2)
        assert cur <= prev * (1 + 1e-12)
        prev = cur
    # and with decay strictly below one the norm strictly shrinks
    assert prev < np.linalg.norm(S0[0, 0], 2)


def pin_split_invariance(run, seed=9):
    """Running T1 tokens, then T2 more tokens from the resulting state, equals
    running T1 + T2 tokens at once (the state is the whole carried memory)."""
    rng = np.random.default_rng(seed)
    T1, T2, H, dk, dv = 5, 7, 2, 4, 3
    q, k, v, la, b = _rand_case(rng, T1 + T2, H, dk, dv)
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = run(q, k, v, la, b, _single(T1 + T2), S0)
    oa, Sa = run(q[:T1], k[:T1], v[:T1], la[:T1], b[:T1], _single(T1), S0)
    ob, Sb = run(q[T1:], k[T1:], v[T1:], la[T1:], b[T1:], _single(T2), Sa)
    assert rel_err(np.concatenate([oa, ob]), o) < RTOL
    assert rel_err(Sb, S) < RTOL


def pin_varlen_independence(run, seed=10):
    """Sequences packed with cu_seqlens do not interact; a zero-length sequence
    returns its initial state unchanged."""
    rng = np.random.default_rng(seed)
    lens = [3, 0, 6, 1]
    T, H, dk, dv = sum(lens), 2, 4, 5
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv)
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    o, S = run(q, k, v, la, b, cu, S0)
    for n, L in enumerate(lens):
        s, e = cu[n], cu[n + 1]
        if L == 0:
            assert np.array_equal(S[n], S0[n])
            continue
        on, Sn = run(q[s:e], k[s:e], v[s:e], la[s:e], b[s:e], _single(L), S0[n:n + 1])
        assert rel_err(o[s:e], on) < RTOL
        assert rel_err(S[n], Sn[0]) < RTOL


def pin_zero_decay_erases_state(run, seed=11):
    """alpha in [0,1] (the KDA section's channel-wise decay bullet) includes 0.  A token
    whose decay is 0 in every key channel (log alpha = -inf) zeroes Diag(alpha_t) S_{t-1},
    so S_t = beta_t k_t v_t^T and o_t = beta_t (q_t . k_t) v_t whatever came before, and
    every later output and the final state are independent of S0 and of the earlier
    tokens.  No value may be NaN or infinite."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv, t0 = 9, 2, 4, 3, 4
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv)
    la[t0] = -np.inf
    cu = _single(T)
    o, S = run(q, k, v, la, b, cu, rng.standard_normal((1, H, dk, dv)))
    assert np.isfinite(o).all() and np.isfinite(S).all()
    for h in range(H):
        want = b[t0, h] * np.dot(q[t0, h], k[t0, h]) * v[t0, h]
        assert rel_err(o[t0, h], want) < RTOL
    _, St0 = run(q[:t0 + 1], k[:t0 + 1], v[:t0 + 1], la[:t0 + 1], b[:t0 + 1], _single(t0 + 1),
                 rng.standard_normal((1, H, dk, dv)))
    for h in range(H):
        assert rel_err(St0[0, h], b[t0, h] * np.outer(k[t0, h], v[t0, h])) < RTOL
    # other earlier tokens and another initial state: the same outputs from t0 on
    q2, k2, v2, la2, b2 = _rand_case(rng, T, H, dk, dv)
    for x, x2 in ((q, q2), (k, k2), (v, v2), (la, la2), (b, b2)):
        x2[t0:] = x[t0:]
    o2, S2 = run(q2, k2, v2, la2, b2, cu, rng.standard_normal((1, H, dk, dv)))
    assert rel_err(o2[t0:], o[t0:]) < RTOL
    assert rel_err(S2, S) < RTOL


def pin_bruteforce_strong_decay(run, seed=12):
    """The explicit products M_t = (I - beta_t k_t k_t^T) Diag(alpha_t) with decays over the
    whole range [0, 1]: single channels with alpha = 0 (log alpha = -inf), decays far below
    the fp32 range (log alpha = -200) and near-one decays mixed in one head."""
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 7, 1, 4, 3
    q, k, v, la, b = _rand_case(rng, T, H, dk, dv, unit_k=False)
    la[:, 0, 0] = -200.0          # channel 0 forgets within one token
    la[2, 0, 1] = -np.inf         # channel 1 is erased at token 2
    la[5, 0, 2] = -np.inf         # channel 2 at token 5
    la[:, 0, 3] = -1e-3           # channel 3 nearly keeps everything
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = run(q, k, v, la, b, _single(T), S0)
    assert np.isfinite(o).all() and np.isfinite(S).all()
    M = [(np.eye(dk) - b[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(la[t, 0])) for t in range(T)]
    St = S0[0, 0]
    for t in range(T):
        St = M[t] @ St + b[t, 0] * np.outer(k[t, 0], v[t, 0])
        assert rel_err(o[t, 0], St.T @ q[t, 0]) < RTOL
    assert rel_err(S[0, 0], St) < RTOL


ALL_PINS = [pin_hand_worked, pin_beta_zero_closed_form, pin_exact_reconstruction,
            pin_orthonormal_linear_attention, pin_scalar_gate_gdn,
            lambda run: pin_scalar_gate_gdn(run, ungated=True),
            pin_bruteforce_products, pin_scalar_d1, pin_linearity,
            pin_householder_norms, pin_split_invariance, pin_varlen_independence,
            pin_zero_decay_erases_state, pin_bruteforce_strong_decay]
