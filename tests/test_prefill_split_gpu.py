"""The tensor-core prefill's sequence split (pass A, the chain of start states, pass B)
against the fp64 oracle and against the same call run without the split; needs a GPU."""
import torch
import pytest

from gated_delta_rule_126_b200 import inputs, kda_prefill, prefill_workspace_size
from tests.kda_check import TOL, compare_full, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(inp, workspace=None):
    return kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"],
                       inp["cu_seqlens_host"], S0=inp["S0"], workspace=workspace)


def _minimal_workspace(n):
    # the status word and the ordering only: too small for the split, so the call runs unsplit
    return torch.zeros(256 + ((4 * n + 255) // 256) * 256, dtype=torch.uint8, device=DEV)


def test_one_long_sequence_is_split():
    """40,000 + 300 + 1,000 tokens, 2 heads, non-zero S0: the long sequence is cut into
    segments (eight at 2 heads); every output and final state is compared with the oracle."""
    inp = inputs.prefill_inputs([40000, 300, 1000], 2, 128, 128, "bf16", s0_std=0.1, seed=51, device=DEV)
    assert prefill_workspace_size(3, 41300, 2, 128, 128) > _minimal_workspace(3).numel()
    o, S = _run(inp)
    torch.cuda.synchronize()
    compare_full(inp, o, S, "bf16")


def test_two_long_sequences_are_split():
    inp = inputs.prefill_inputs([20000, 5, 18000], 1, 128, 128, "bf16", s0_std=0.1, seed=52, device=DEV)
    o, S = _run(inp)
    torch.cuda.synchronize()
    compare_full(inp, o, S, "bf16")


def test_split_agrees_with_the_unsplit_run():
    """Same inputs through a minimum workspace (no room for the split): the results agree
    within the bf16 bounds, and the short sequence, which is never split, bit for bit."""
    inp = inputs.prefill_inputs([33000, 700], 2, 128, 128, "bf16", s0_std=0.1, seed=53, device=DEV)
    o1, S1 = _run(inp)
    o2, S2 = _run(inp, workspace=_minimal_workspace(2))
    torch.cuda.synchronize()
    assert rel_l2(host64(o1), host64(o2)) <= TOL["bf16"]["o"]
    assert rel_l2(host64(S1), host64(S2)) <= TOL["bf16"]["S"]
    assert torch.equal(o1[33000:], o2[33000:]) and torch.equal(S1[1], S2[1])


def test_few_heads_take_more_segments():
    """60,000 + 300 tokens on 2 heads: pass A's units leave room for the most segments
    (eight, one start-state chain step each past the second); against the oracle, and the
    short sequence bit for bit against the unsplit run."""
    inp = inputs.prefill_inputs([60000, 300], 2, 128, 128, "bf16", s0_std=0.1, seed=54, device=DEV)
    o, S = _run(inp)
    o2, S2 = _run(inp, workspace=_minimal_workspace(2))
    torch.cuda.synchronize()
    compare_full(inp, o, S, "bf16")
    assert torch.equal(o[60000:], o2[60000:]) and torch.equal(S[1], S2[1])


def test_two_sequences_share_the_segments():
    """Two long sequences on one head, eight segments each, and a short one."""
    inp = inputs.prefill_inputs([40000, 100, 36000], 1, 128, 128, "bf16", s0_std=0.1, seed=55, device=DEV)
    o, S = _run(inp)
    torch.cuda.synchronize()
    compare_full(inp, o, S, "bf16")
