"""Parity of kda_prologue (short conv, Swish, L2Norm, gates) with its fp64 oracle, and of
the chain prologue -> prefill with the oracles chained the same way; needs a GPU."""
import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as pro
from gated_delta_rule_126_b200 import inputs, kda_prefill, kda_prologue
from tests.kda_check import TOL, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


def _run(p, eps=EPS):
    return kda_prologue(p["q_pre"], p["k_pre"], p["v_pre"], p["conv_q"], p["conv_k"], p["conv_v"],
                        p["a_gate"], p["rate"], p["b_gate"], p["cu_seqlens"],
                        cu_seqlens_host=p["cu_seqlens_host"], l2_eps=eps)


def _oracle(p, eps=EPS, seqs=None):
    """Oracle outputs; ``seqs`` restricts them to some sequences (returned as row slices)."""
    cu = p["cu_seqlens_host"]
    idx = range(len(cu) - 1) if seqs is None else seqs
    outs = {}
    for n in idx:
        s, e = cu[n], cu[n + 1]
        sl = lambda t: host64(t[s:e])
        outs[n] = pro.prologue(sl(p["q_pre"]), sl(p["k_pre"]), sl(p["v_pre"]), host64(p["conv_q"]),
                               host64(p["conv_k"]), host64(p["conv_v"]), sl(p["a_gate"]), host64(p["rate"]),
                               sl(p["b_gate"]), [0, e - s], eps=eps)
    return outs


def _check(p, out, dtype, seqs=None):
    cu = p["cu_seqlens_host"]
    tol = TOL[dtype]["o"]
    for n, (q, k, v, la, beta) in _oracle(p, seqs=seqs).items():
        s, e = cu[n], cu[n + 1]
        if e == s:
            continue
        for name, ref in (("q", q), ("k", k), ("v", v)):
            err = rel_l2(host64(out[name][s:e]), ref)
            assert err <= tol, (n, name, err)
        assert rel_l2(host64(out["log_alpha"][s:e]), la) <= 1e-6
        assert rel_l2(host64(out["beta"][s:e]), beta) <= 1e-6


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 128), ("f32", 16, 8), ("bf16", 32, 64)])
@pytest.mark.parametrize("width", [1, 2, 4])
def test_ragged_varlen(dtype, dk, dv, width):
    """Sequences of length 0, 1, 2, 3, 5 and 70 packed: the convolution restarts at each start."""
    p = inputs.prologue_inputs([3, 0, 1, 70, 2, 5], 3, dk, dv, dtype, width=width, seed=41, device=DEV)
    out = _run(p)
    torch.cuda.synchronize()
    _check(p, out, dtype)


def test_batched_workload_sampled():
    """The batched workload's shape (8 x 8192 tokens, 32 heads, bf16); three sequences in full."""
    p = inputs.prologue_inputs([8192] * 8, 32, 128, 128, "bf16", width=4, seed=42, device=DEV)
    out = _run(p)
    torch.cuda.synchronize()
    _check(p, out, "bf16", seqs=[0, 3, 7])
    # properties at full size: q, k rows have unit norm (to bf16 rounding); log alpha <= 0
    nq = out["q"].float().norm(dim=-1)
    assert torch.allclose(nq, torch.ones_like(nq), atol=1e-2)
    assert bool((out["log_alpha"] <= 0).all())


def test_chain_prologue_then_prefill():
    """prologue -> kda_prefill on the GPU.  The prefill is held to its usual bf16 bound
    against the oracle recurrence run on the prologue's own (bf16) outputs, the prologue to
    its bound above.  Against the all-fp64 chain (oracle prologue, then oracle recurrence)
    o also carries the bf16 rounding of q, k and v (about 2^-9 / sqrt(3) relative each), so
    that comparison gets the bound 5e-3."""
    lens = [200, 64, 1, 130]
    p = inputs.prologue_inputs(lens, 4, 128, 128, "bf16", width=4, seed=43, device=DEV)
    out = _run(p)
    o, S = kda_prefill(out["q"], out["k"], out["v"], out["log_alpha"], out["beta"], p["cu_seqlens"],
                       p["cu_seqlens_host"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.prefill(host64(out["q"]), host64(out["k"]), host64(out["v"]),
                                  host64(out["log_alpha"]), host64(out["beta"]), p["cu_seqlens_host"])
    assert rel_l2(host64(o), o_ref) <= TOL["bf16"]["o"]
    assert rel_l2(host64(S), S_ref) <= TOL["bf16"]["S"]
    _check(p, out, "bf16")
    q, k, v, la, beta = (np.concatenate([x[i] for x in _oracle(p).values()]) for i in range(5))
    o64, S64 = oracle.prefill(q, k, v, la, beta, p["cu_seqlens_host"])
    assert rel_l2(host64(o), o64) <= 5e-3
    assert rel_l2(host64(S), S64) <= 5e-3
