"""Parity of the CUDA decode step with the fp64 oracle (needs a GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_126_b200 import inputs, kda_decode_step
from tests.kda_check import TOL, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_steps(inp, steps):
    S = inp["S0"].clone()
    outs = []
    for t in range(steps):
        outs.append(kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["log_alpha"][t],
                                    inp["beta"][t], S))
    torch.cuda.synchronize()
    return torch.stack(outs), S


def _oracle_unit(inp, b, h, steps):
    """``steps`` decode steps of one (sequence, head) = a prefill of that many tokens."""
    sl = lambda x: host64(x[:steps, b, h:h + 1])
    o, S = oracle.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                          host64(inp["beta"][:steps, b, h:h + 1]), [0, steps],
                          S0=host64(inp["S0"][b:b + 1, h:h + 1]))
    return o[:, 0], S[0, 0]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (16, 8), (37, 44), (128, 64)])
def test_decode_small(dtype, dk, dv):
    B, H, steps = 3, 2, 6
    inp = inputs.decode_inputs(B, H, dk, dv, steps, dtype, seed=7, device=DEV)
    o, S = _run_steps(inp, steps)
    worst_o = worst_S = 0.0
    for b in range(B):
        for h in range(H):
            o_ref, S_ref = _oracle_unit(inp, b, h, steps)
            worst_o = max(worst_o, rel_l2(host64(o[:, b, h]), o_ref))
            worst_S = max(worst_S, rel_l2(host64(S[b, h]), S_ref))
    assert worst_o <= TOL[dtype]["o"] and worst_S <= TOL[dtype]["S"], (worst_o, worst_S)


def test_decode_full_workload_sampled():
    """256 sequences x 32 heads, d = 128, 64 consecutive steps (the decode workload),
    checked on sampled (sequence, head) pairs over all 64 steps."""
    w = inputs.WORKLOADS["decode"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, S = _run_steps(inp, w.steps)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    rng = np.random.default_rng(0)
    units = {(0, 0), (w.batch - 1, w.H - 1)}
    units |= {(int(rng.integers(w.batch)), int(rng.integers(w.H))) for _ in range(30)}
    worst_o = worst_S = 0.0
    for b, h in sorted(units):
        o_ref, S_ref = _oracle_unit(inp, b, h, w.steps)
        worst_o = max(worst_o, rel_l2(host64(o[:, b, h]), o_ref))
        worst_S = max(worst_S, rel_l2(host64(S[b, h]), S_ref))
    assert worst_o <= TOL["bf16"]["o"] and worst_S <= TOL["bf16"]["S"], (worst_o, worst_S)


def test_decode_zero_batch_is_noop():
    q = torch.empty(0, 2, 128, dtype=torch.bfloat16, device=DEV)
    v = torch.empty(0, 2, 128, dtype=torch.bfloat16, device=DEV)
    la = torch.empty(0, 2, 128, device=DEV)
    b = torch.empty(0, 2, device=DEV)
    S = torch.empty(0, 2, 128, 128, device=DEV)
    o = kda_decode_step(q, q, v, la, b, S)
    assert o.shape == (0, 2, 128)
