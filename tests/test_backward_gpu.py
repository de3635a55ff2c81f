"""Parity of the CUDA backward pass with the fp64 adjoint oracle (needs a GPU).

The oracle (``oracle.backward``) runs the exact reverse-mode sweep of the token
recurrence in fp64 and is pinned by central finite differences of the forward
oracle.  The kernels compute in float32 from the same (bf16-rounded where the
inputs are bf16) values, so every gradient is held to relative L2 <= 1e-5, the
fp32 bound of the forward parity tests (a float32 model of the same algorithm
lands near 3e-7, at 1024 tokens as at 64).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_126_b200 import inputs, kda_backward
from tests.kda_check import host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-5
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def run_gpu(inp, dO, dS, **kw):
    return kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"], dO,
                        cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"], dS_final=dS, **kw)


def run_oracle(inp, dO, dS):
    S0 = None if inp["S0"] is None else host64(inp["S0"])
    return oracle.backward(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), host64(inp["log_alpha"]),
                           host64(inp["beta"]), inp["cu_seqlens_host"], host64(dO), S0=S0,
                           dS_final=None if dS is None else host64(dS))


def check_all(got, ref, names=NAMES):
    errs = {n: rel_l2(host64(got[n]), ref[n]) for n in names}
    bad = {n: e for n, e in errs.items() if not e <= TOL}
    assert not bad, errs


def case(seqlens, H, dk, dv, dtype, s0=0.1, ds=0.1, seed=5):
    inp = inputs.prefill_inputs(seqlens, H, dk, dv, dtype, s0_std=s0, seed=seed, device=DEV)
    dO, dS = inputs.grad_inputs(sum(seqlens), len(seqlens), H, dk, dv, dtype, seed=seed + 1, device=DEV,
                                ds_std=ds)
    return inp, dO, dS


def test_tiny_f32():
    """B=1, H=1, T=64, d=16, fp32, with S0 and dS_final."""
    inp, dO, dS = case([64], 1, 16, 16, "f32")
    check_all(run_gpu(inp, dO, dS), run_oracle(inp, dO, dS))


@pytest.mark.parametrize("dtype,dk,dv", [("f32", 16, 20), ("bf16", 7, 5), ("f32", 32, 48), ("bf16", 128, 128),
                                         ("bf16", 128, 100), ("f32", 128, 17)])
def test_ragged_varlen(dtype, dk, dv):
    """Empty, one-token, checkpoint-aligned, one-past and ragged lengths packed together;
    value widths that fill a slice, part of one, and several."""
    inp, dO, dS = case([1, 17, 0, 32, 33, 70, 5], 2, dk, dv, dtype)
    check_all(run_gpu(inp, dO, dS), run_oracle(inp, dO, dS))


def test_without_initial_state_or_final_gradient():
    """S0 = 0, dS_final = 0, dS0 not requested."""
    inp, dO, dS = case([40, 9], 3, 128, 128, "bf16", s0=0.0, ds=0.0)
    got = run_gpu(inp, dO, dS, want_dS0=False)
    assert got["dS0"] is None
    check_all(got, run_oracle(inp, dO, dS), NAMES[:-1])


def test_single_sequence_workload():
    """B=1, H=4, T=4096, d=128, bf16 q/k/v/dO: every gradient element compared."""
    w = inputs.WORKLOADS["single_seq_prefill"]
    inp = inputs.workload_inputs(w, device=DEV)
    dO, dS = inputs.grad_inputs(4096, 1, w.H, w.dk, w.dv, w.dtype, seed=w.seed + 100, device=DEV)
    check_all(run_gpu(inp, dO, dS), run_oracle(inp, dO, dS))


def test_alpha1_beta0_closed_form():
    """alpha = 1, beta = 0: the state never moves (S_t = S0), so dq_t = S0 do_t,
    dk = dv = 0, dS0 = dS_final + sum_t q_t do_t^T, dbeta_t = k_t^T G_t (v_t - S0^T k_t) with
    G_t = dS_final + sum_{tau >= t} q_tau do_tau^T, and dlog_alpha_t[i] = (G_t S0^T)_ii
    -- written out in fp64 here, independent of the oracle."""
    inp, dO, dS = case([50], 1, 16, 24, "f32", seed=9)
    inp["log_alpha"].zero_()
    inp["beta"].zero_()
    got = run_gpu(inp, dO, dS)
    q, k, v, do = (host64(t[:, 0]) for t in (inp["q"], inp["k"], inp["v"], dO))
    S0, dSf = host64(inp["S0"][0, 0]), host64(dS[0, 0])
    G = np.empty((50, 16, 24))
    acc = dSf.copy()
    for t in range(49, -1, -1):
        acc = acc + np.outer(q[t], do[t])
        G[t] = acc
    ref = dict(dq=(do @ S0.T)[:, None], dk=np.zeros((50, 1, 16)), dv=np.zeros((50, 1, 24)),
               dS0=acc[None, None], dbeta=np.einsum("ti,tij,tj->t", k, G, v - k @ S0)[:, None],
               dlog_alpha=np.einsum("tij,ij->ti", G, S0)[:, None])
    for n in ("dq", "dS0", "dbeta", "dlog_alpha"):
        assert rel_l2(host64(got[n]), ref[n]) <= TOL, n
    for n in ("dk", "dv"):
        assert float(got[n].abs().max()) == 0.0, n


def test_bench_size_sampled_units():
    """The 2 x 8192, H = 32 bf16 batch the bench times: four (sequence, head) units
    compared in full against the oracle run on that unit alone."""
    w = inputs.WORKLOADS["batched_prefill_2x8192"]
    inp = inputs.workload_inputs(w, device=DEV)
    T = inp["q"].shape[0]
    N = len(inp["cu_seqlens_host"]) - 1
    dO, dS = inputs.grad_inputs(T, N, w.H, w.dk, w.dv, w.dtype, seed=w.seed + 100, device=DEV)
    got = run_gpu(inp, dO, dS)
    cu = inp["cu_seqlens_host"]
    for n, h in [(0, 0), (1, 31), (0, 17), (1, 5)]:
        s, e = cu[n], cu[n + 1]
        sub = {key: inp[key][s:e, h:h + 1] for key in ("q", "k", "v", "log_alpha", "beta")}
        sub["S0"] = inp["S0"][n:n + 1, h:h + 1] if inp["S0"] is not None else None
        sub["cu_seqlens_host"] = [0, e - s]
        ref = run_oracle(sub, dO[s:e, h:h + 1], dS[n:n + 1, h:h + 1])
        part = {key: got[key][s:e, h:h + 1] for key in NAMES[:-1]}
        part["dS0"] = got["dS0"][n:n + 1, h:h + 1]
        check_all(part, ref)


def test_empty_sequences_pass_the_final_gradient_through():
    """Empty sequences among non-empty ones: their dS0 is dS_final unchanged, and the
    non-empty ones match the oracle."""
    inp, dO, dS = case([0, 5, 0, 40, 0], 2, 32, 24, "f32", seed=11)
    got = run_gpu(inp, dO, dS)
    for n in (0, 2, 4):
        assert torch.equal(got["dS0"][n], dS[n])
    check_all(got, run_oracle(inp, dO, dS))


def test_all_sequences_empty():
    """T = 0: no token gradients exist; dS0 = dS_final."""
    inp, dO, dS = case([0, 0], 1, 16, 16, "f32", seed=12)
    got = run_gpu(inp, dO, dS)
    assert got["dq"].numel() == 0 and got["dbeta"].numel() == 0
    assert torch.equal(got["dS0"], dS)
