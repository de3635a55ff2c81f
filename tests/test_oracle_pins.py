"""The fp64 oracle and the fp64 chunk model against the pins in ``pins.py``."""
import numpy as np
import pytest

import oracle
from oracle import chunk_model
from tests import pins


def run_oracle(q, k, v, la, b, cu, S0):
    return oracle.prefill(q, k, v, la, b, cu, S0=S0)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: getattr(p, "__name__", "pin"))
def test_oracle_pin(pin):
    pin(run_oracle)


@pytest.mark.parametrize("chunk", [1, 3, 4, 64])
@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: getattr(p, "__name__", "pin"))
def test_chunk_model_pin(pin, chunk):
    pin(lambda q, k, v, la, b, cu, S0: chunk_model.prefill(q, k, v, la, b, cu, S0=S0, chunk=chunk))


@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_chunk_model_matches_recurrence(chunk):
    """The chunk rewrite equals the token recurrence to fp64 rounding, with ragged
    last chunks, d_k != d_v, several sequences and a non-zero initial state."""
    rng = np.random.default_rng(11)
    lens = [37, 1, 64, 0, 70]
    T, H, dk, dv = sum(lens), 2, 12, 7
    q, k, v, la, b = pins._rand_case(rng, T, H, dk, dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    o_ref, S_ref = oracle.prefill(q, k, v, la, b, cu, S0=S0)
    o, S = chunk_model.prefill(q, k, v, la, b, cu, S0=S0, chunk=chunk)
    assert pins.rel_err(o, o_ref) < 1e-12
    assert pins.rel_err(S, S_ref) < 1e-12


def test_chunk_stage_identities():
    """Stage values of one chunk satisfy their defining equations: (I + A) T =
    Diag(beta) with I + A unit lower triangular, P lower triangular including
    the diagonal, and U = T (V - (K*exp(g)) S) solves (I + A) U = Diag(beta)(V - (K*exp(g)) S)."""
    rng = np.random.default_rng(12)
    L, dk, dv = 16, 8, 6
    q, k, v, la, b = (x[:, 0] for x in pins._rand_case(rng, L, 1, dk, dv))
    st = chunk_model.chunk_stages(q, k, v, la, b[:, 0] if b.ndim == 2 else b)
    A, T, P = st["A"], st["T"], st["P"]
    assert np.allclose(np.triu(A), 0)
    assert np.allclose(np.triu(P, 1), 0)
    beta = b[:, 0] if b.ndim == 2 else b
    assert np.allclose((np.eye(L) + A) @ T, np.diag(beta), atol=1e-13)
    S = rng.standard_normal((dk, dv))
    _, _, U = chunk_model.chunk_step(st, S)
    rhs = beta[:, None] * (v - st["Kg"] @ S)
    assert np.allclose((np.eye(L) + A) @ U, rhs, atol=1e-12)


def test_oracle_thread_count_invariant():
    rng = np.random.default_rng(13)
    lens = [20, 9, 33]
    T, H, dk, dv = sum(lens), 3, 6, 5
    q, k, v, la, b = pins._rand_case(rng, T, H, dk, dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o1, S1 = oracle.prefill(q, k, v, la, b, cu, nthreads=1)
    o4, S4 = oracle.prefill(q, k, v, la, b, cu, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)


def test_oracle_decode_is_length_one_prefill():
    rng = np.random.default_rng(14)
    B, H, dk, dv = 5, 2, 4, 3
    q, k, v, la, b = pins._rand_case(rng, B, H, dk, dv)
    S = rng.standard_normal((B, H, dk, dv))
    o, S1 = oracle.decode_step(q, k, v, la, b, S)
    for n in range(B):
        on, Sn = oracle.prefill(q[n:n + 1], k[n:n + 1], v[n:n + 1], la[n:n + 1], b[n:n + 1],
                                [0, 1], S0=S[n:n + 1])
        assert np.array_equal(on, o[n:n + 1]) and np.array_equal(Sn[0], S1[n])


def test_oracle_rejects_bad_cu_seqlens():
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, q, np.zeros((4, 1)), [0, 3, 2, 4])
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, q, np.zeros((4, 1)), [0, 3])
