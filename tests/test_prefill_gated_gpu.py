"""Parity of kda_prefill_gated (prefill + sigmoid output gate + RMSNorm) with the fp64
oracles (the recurrence, then the epilogue); needs a GPU."""
import numpy as np
import pytest
import torch

import oracle
from oracle import epilogue
from gated_delta_rule_126_b200 import inputs, kda_prefill, kda_prefill_gated
from tests.kda_check import TOL, host64, oracle_units, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


def _inputs(lens, H, dk, dv, dtype, s0_std=0.1, seed=31):
    inp = inputs.prefill_inputs(lens, H, dk, dv, dtype, s0_std=s0_std, seed=seed, device=DEV)
    gate, w = inputs.gate_inputs(sum(lens), H, dv, dtype, seed=seed + 1, device=DEV)
    return inp, gate, w


def _run(inp, gate, w, chunk=64, eps=EPS):
    return kda_prefill_gated(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             inp["cu_seqlens"], gate, w, eps, cu_seqlens_host=inp["cu_seqlens_host"],
                             S0=inp["S0"], chunk=chunk)


def _oracle_all(inp, gate, w, eps=EPS):
    o, S = oracle.prefill(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]),
                          host64(inp["log_alpha"]), host64(inp["beta"]), inp["cu_seqlens_host"],
                          S0=None if inp["S0"] is None else host64(inp["S0"]))
    return epilogue.gated_rmsnorm(o, host64(gate), host64(w), eps), S


@pytest.mark.parametrize("dtype,dk,dv,chunk", [("bf16", 128, 128, 64), ("f32", 16, 16, 16),
                                               ("f32", 32, 48, 32), ("f32", 128, 128, 64)])
def test_ragged_varlen(dtype, dk, dv, chunk):
    """Empty, one-token, one-chunk, chunk-plus-one and multi-chunk sequences with a ragged
    tail, packed; a non-zero initial state.  bf16 runs the fused tensor-core epilogue,
    float32 the prefill followed by the in-place epilogue kernel."""
    lens = [1, 17, 64, 65, 0, 130, 3]
    inp, gate, w = _inputs(lens, 3, dk, dv, dtype)
    y, S = _run(inp, gate, w, chunk=chunk)
    torch.cuda.synchronize()
    y_ref, S_ref = _oracle_all(inp, gate, w)
    tol = TOL[dtype]
    ey, eS = rel_l2(host64(y), y_ref), rel_l2(host64(S), S_ref)
    assert ey <= tol["o"] and eS <= tol["S"], (ey, eS)


def test_state_path_unchanged_by_the_epilogue():
    """S_final of the gated call equals kda_prefill's bit for bit (same state path), and y
    equals the epilogue applied to kda_prefill's o within the bf16 bound."""
    lens = [300, 64, 1000]
    inp, gate, w = _inputs(lens, 4, 128, 128, "bf16")
    y, S = _run(inp, gate, w)
    o, S2 = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                        inp["cu_seqlens"], inp["cu_seqlens_host"], S0=inp["S0"])
    torch.cuda.synchronize()
    assert torch.equal(S, S2)
    y_from_o = epilogue.gated_rmsnorm(host64(o), host64(gate), host64(w), EPS)
    assert rel_l2(host64(y), y_from_o) <= TOL["bf16"]["o"]


def test_saturated_gate_unit_weight_gives_unit_rms():
    """With the gate saturated (sigmoid = 1), w = 1 and a tiny eps, every stored row has
    mean square 1 -- a property that holds at any size."""
    lens = [8192, 4096]
    inp, gate, w = _inputs(lens, 8, 128, 128, "bf16", s0_std=0.0)
    gate.fill_(30.0)
    w.fill_(1.0)
    y, _ = _run(inp, gate, w, eps=1e-12)
    ms = y.float().pow(2).mean(-1)
    torch.cuda.synchronize()
    assert torch.allclose(ms, torch.ones_like(ms), rtol=0, atol=1.2e-2), float((ms - 1).abs().max())


def test_batched_workload_sampled():
    """The batched workload (8 x 8192 tokens, 32 heads) in the launch bench.py times;
    (sequence, head) units sampled and compared with the oracles one by one."""
    w_ = inputs.WORKLOADS["batched_prefill"]
    inp = inputs.workload_inputs(w_, device=DEV)
    gate, wt = inputs.gate_inputs(w_.total_tokens, w_.H, w_.dv, "bf16", seed=w_.seed + 7, device=DEV)
    y, S = _run(inp, gate, wt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    units = [(int(rng.integers(len(w_.seqlens))), int(rng.integers(w_.H))) for _ in range(4)]
    ref = oracle_units(inp, units, w_.H)
    cu = inp["cu_seqlens_host"]
    worst_y = worst_S = 0.0
    for (n, h), (o_ref, S_ref) in ref.items():
        s, e = cu[n], cu[n + 1]
        y_ref = epilogue.gated_rmsnorm(o_ref, host64(gate[s:e, h]), host64(wt), EPS)
        worst_y = max(worst_y, rel_l2(host64(y[s:e, h]), y_ref))
        worst_S = max(worst_S, rel_l2(host64(S[n, h]), S_ref))
    assert worst_y <= TOL["bf16"]["o"] and worst_S <= TOL["bf16"]["S"], (worst_y, worst_S)


def test_long_sequence_is_split():
    """A 24,000-token sequence next to a 500-token one, 2 heads: the gated call cuts the long
    sequence into segments as kda_prefill does (the segment passes that produce no outputs
    load no gate tiles).  y and S_final against the oracles; S_final bit for bit against
    kda_prefill, which takes the same state path."""
    inp, gate, w = _inputs([24000, 500], 2, 128, 128, "bf16", seed=37)
    y, S = _run(inp, gate, w)
    o_p, S_p = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"],
                           inp["cu_seqlens_host"], S0=inp["S0"])
    torch.cuda.synchronize()
    assert torch.equal(S, S_p)
    y_ref, S_ref = _oracle_all(inp, gate, w)
    ey, eS = rel_l2(host64(y), y_ref), rel_l2(host64(S), S_ref)
    assert ey <= TOL["bf16"]["o"] and eS <= TOL["bf16"]["S"], (ey, eS)
