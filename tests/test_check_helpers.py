"""The GPU parity helpers catch what they are meant to catch (no GPU needed): the oracle's
own outputs pass, and a small error planted in one head, one sequence or one token fails."""
import pytest
import torch

import oracle
from gated_delta_rule_126_b200 import inputs
from tests.kda_check import TOL, compare_heads, compare_units, host64


@pytest.fixture(scope="module")
def case():
    inp = inputs.prefill_inputs([5, 0, 70, 33], 4, 16, 16, "f32", s0_std=0.1, seed=3, device="cpu")
    o, S = oracle.prefill(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), host64(inp["log_alpha"]),
                          host64(inp["beta"]), inp["cu_seqlens_host"], S0=host64(inp["S0"]))
    return inp, torch.from_numpy(o), torch.from_numpy(S)


def test_oracle_outputs_pass(case):
    inp, o, S = case
    eo, eS = compare_heads(inp, o, S, [0, 2, 3], "f32")
    assert eo < 1e-12 and eS < 1e-12
    compare_units(inp, o, S, [(0, 1), (2, 3), (3, 0)], "f32")


@pytest.mark.parametrize("where", ["S of one sequence", "o of one token", "o of the last row"])
def test_planted_error_fails(case, where):
    inp, o, S = case
    o, S = o.clone(), S.clone()
    if where == "S of one sequence":
        S[2, 3] *= 1 + 1e-3
    elif where == "o of one token":
        o[40, 3] += 1e-2 * float(o[40, 3].abs().max())
    else:
        o[-1, 3] = -o[-1, 3]
    with pytest.raises(AssertionError):
        compare_heads(inp, o, S, [0, 3], "f32")


def test_error_outside_the_heads_compared_is_not_seen(case):
    """compare_heads checks only the heads it is given (the full-size tests pick three)."""
    inp, o, S = case
    S = S.clone()
    S[:, 1] += 1.0
    compare_heads(inp, o, S, [0, 2, 3], "f32")
    with pytest.raises(AssertionError):
        compare_heads(inp, o, S, [1], "f32")


def test_tolerances_are_the_stated_ones():
    """The bounds every parity test uses: rel-L2 1e-5 for float32 q/k/v, and 3e-3 on o and
    1e-3 on S for bfloat16 q/k/v with a float32 state."""
    assert TOL["f32"] == dict(o=1e-5, S=1e-5) and TOL["bf16"] == dict(o=3e-3, S=1e-3)
