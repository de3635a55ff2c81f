"""Pins of the fp64 backward oracle: central finite differences of the forward oracle.

The forward oracle is itself pinned (tests/pins.py); differentiating it numerically
is independent of the adjoint sweep, so every gradient the adjoint returns is checked
against an estimate that shares none of its code.  With h = 1e-5 in fp64 the central
difference is exact to about 1e-9 relative on these sizes.
"""
import numpy as np
import pytest

import oracle


def _case(seed, lens=(5, 0, 9), H=2, dk=3, dv=4, s0=True):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -0.3 * np.log1p(np.exp(rng.standard_normal((T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = rng.standard_normal((len(lens), H, dk, dv)) if s0 else None
    dO = rng.standard_normal((T, H, dv))
    dS = rng.standard_normal((len(lens), H, dk, dv))
    return dict(q=q, k=k, v=v, la=la, b=b, cu=cu, S0=S0, dO=dO, dS=dS)


def _loss(c, **over):
    x = {**c, **over}
    o, S = oracle.prefill(x["q"], x["k"], x["v"], x["la"], x["b"], x["cu"], S0=x["S0"])
    return float(np.sum(o * c["dO"]) + np.sum(S * c["dS"]))


def _fd(c, name, h=1e-5):
    base = c[name]
    g = np.zeros_like(base)
    it = np.nditer(base, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        p, m = base.copy(), base.copy()
        p[i] += h
        m[i] -= h
        g[i] = (_loss(c, **{name: p}) - _loss(c, **{name: m})) / (2 * h)
    return g


@pytest.mark.parametrize("name,key", [("q", "dq"), ("k", "dk"), ("v", "dv"), ("la", "dlog_alpha"),
                                      ("b", "dbeta"), ("S0", "dS0")])
def test_gradient_matches_finite_differences(name, key):
    c = _case(1)
    g = oracle.backward(c["q"], c["k"], c["v"], c["la"], c["b"], c["cu"], c["dO"], S0=c["S0"], dS_final=c["dS"])
    fd = _fd(c, name)
    err = np.linalg.norm(g[key] - fd) / np.linalg.norm(fd)
    assert err < 1e-7, (name, err)


def test_no_initial_state_and_no_final_gradient():
    c = _case(2, lens=(7, 4), s0=False)
    c["dS"] = np.zeros_like(c["dS"])
    g = oracle.backward(c["q"], c["k"], c["v"], c["la"], c["b"], c["cu"], c["dO"])
    for name, key in (("k", "dk"), ("la", "dlog_alpha")):
        fd = _fd(c, name)
        assert np.linalg.norm(g[key] - fd) / np.linalg.norm(fd) < 1e-7


def test_long_sequence_crosses_checkpoints():
    # 150 tokens: the adjoint recomputes states from checkpoints every 64 tokens
    c = _case(3, lens=(150,), H=1, dk=2, dv=2)
    g = oracle.backward(c["q"], c["k"], c["v"], c["la"], c["b"], c["cu"], c["dO"], S0=c["S0"], dS_final=c["dS"])
    for name, key in (("v", "dv"), ("b", "dbeta"), ("S0", "dS0")):
        fd = _fd(c, name)
        assert np.linalg.norm(g[key] - fd) / np.linalg.norm(fd) < 1e-7, name


def test_linear_attention_special_case():
    # alpha = 1, beta = 0: o_t = S0^T q_t, so dq_t = S0 do_t and dS0 = sum_t q_t do_t^T + dS_final;
    # nothing flows to v or k
    c = _case(4, lens=(6,), H=1)
    c["la"][:] = 0.0
    c["b"][:] = 0.0
    g = oracle.backward(c["q"], c["k"], c["v"], c["la"], c["b"], c["cu"], c["dO"], S0=c["S0"], dS_final=c["dS"])
    S0 = c["S0"][0, 0]
    assert np.allclose(g["dq"][:, 0], c["dO"][:, 0] @ S0.T, rtol=1e-12)
    assert np.allclose(g["dS0"][0, 0], c["q"][:, 0].T @ c["dO"][:, 0] + c["dS"][0, 0], rtol=1e-12)
    assert np.array_equal(g["dv"], np.zeros_like(g["dv"]))
    assert np.array_equal(g["dk"], np.zeros_like(g["dk"]))
    # G_t = dS_final + sum_{tau >= t} q_tau do_tau^T is the gradient of the (unmoving) state
    # after token t; beta_t scales k_t (v_t - S0^T k_t)^T and log alpha_t scales S0's rows
    q, k, v, do = c["q"][:, 0], c["k"][:, 0], c["v"][:, 0], c["dO"][:, 0]
    G = np.cumsum((q[:, :, None] * do[:, None, :])[::-1], axis=0)[::-1] + c["dS"][0, 0]
    assert np.allclose(g["dbeta"][:, 0], np.einsum("ti,tij,tj->t", k, G, v - k @ S0), rtol=1e-12)
    assert np.allclose(g["dlog_alpha"][:, 0], np.einsum("tij,ij->ti", G, S0), rtol=1e-12)


@pytest.mark.parametrize("T,chunk", [(37, 8), (64, 16), (5, 8), (130, 64)])
def test_chunk_backward_model_matches_adjoint(T, chunk):
    """The chunk-form backward (the algorithm the GPU kernel follows) equals the token
    adjoint to fp64 rounding, with ragged last chunks."""
    from oracle import chunk_model
    rng = np.random.default_rng(T)
    dk, dv = 6, 5
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, dv))
    la = -0.2 * np.log1p(np.exp(rng.standard_normal((T, 1, dk))))
    b = 1 / (1 + np.exp(-rng.standard_normal((T, 1))))
    S0 = rng.standard_normal((1, 1, dk, dv))
    dO = rng.standard_normal((T, 1, dv))
    dS = rng.standard_normal((1, 1, dk, dv))
    g = oracle.backward(q, k, v, la, b, [0, T], dO, S0=S0, dS_final=dS)
    r = chunk_model.chunk_backward_unit(q[:, 0], k[:, 0], v[:, 0], la[:, 0], b[:, 0], dO[:, 0], S0[0, 0],
                                        dS[0, 0], chunk=chunk)
    for name, got in zip(["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"], r):
        ref = g[name][0, 0] if name == "dS0" else g[name][:, 0]
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-12, name
