"""Parity of the CUDA chunked prefill with the fp64 oracle (needs a GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_126_b200 import inputs, kda_decode_step, kda_prefill
from tests.kda_check import TOL, compare_full, compare_heads, compare_units, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(inp, chunk=64, S0="inp", **kw):
    return kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       inp["cu_seqlens"], inp["cu_seqlens_host"],
                       S0=inp["S0"] if S0 == "inp" else S0, chunk=chunk, **kw)


def test_tiny_f32_workload():
    """B=1, H=1, T=64, d=16, fp32, chunk 16: whole-tensor rel-L2 <= 1e-5."""
    w = inputs.WORKLOADS["tiny_f32"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, S = run(inp, chunk=w.chunk)
    compare_full(inp, o, S, "f32")


@pytest.mark.parametrize("case", ["alpha1_beta0", "alpha1_beta1"])
def test_tiny_invariant_cases(case):
    """alpha = 1 with beta = 0 (state carried unchanged) and with beta = 1 (pure delta
    rule), on the tiny fp32 shape, with a non-zero initial state."""
    w = inputs.WORKLOADS["tiny_f32"]
    inp = inputs.prefill_inputs(w.seqlens, w.H, w.dk, w.dv, "f32", s0_std=0.1, seed=w.seed,
                                device=DEV)
    inp["log_alpha"].zero_()
    inp["beta"].fill_(0.0 if case == "alpha1_beta0" else 1.0)
    o, S = run(inp, chunk=w.chunk)
    compare_full(inp, o, S, "f32")
    if case == "alpha1_beta0":
        torch.testing.assert_close(S, inp["S0"], rtol=0, atol=1e-6)


def test_single_sequence_prefill_workload():
    """B=1, H=4, T=4096, d=128, bf16 q/k/v, S0 ~ N(0, 0.01): every output compared."""
    w = inputs.WORKLOADS["single_seq_prefill"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, S = run(inp, chunk=w.chunk)
    compare_full(inp, o, S, "bf16")


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 128, 128), ("f32", 32, 48),
                                         ("bf16", 5, 7)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_varlen(dtype, dk, dv, chunk):
    """Lengths that are empty, one token, exactly one chunk, one past a chunk and
    several chunks with a ragged tail, packed together."""
    lens = [1, 17, 64, 65, 0, 130, 3]
    inp = inputs.prefill_inputs(lens, 3, dk, dv, dtype, s0_std=0.1, seed=3, device=DEV)
    o, S = run(inp, chunk=chunk)
    compare_full(inp, o, S, dtype)


def test_chunk_size_invariance():
    lens = [200, 77]
    inp = inputs.prefill_inputs(lens, 2, 64, 64, "f32", s0_std=0.1, seed=4, device=DEV)
    res = [run(inp, chunk=c) for c in (16, 32, 64)]
    for o, S in res[1:]:
        assert rel_l2(host64(o), host64(res[0][0])) < 1e-5
        assert rel_l2(host64(S), host64(res[0][1])) < 1e-5


def test_split_invariance_and_aliasing():
    """prefill(T1) then prefill(T2) from its state equals prefill(T1 + T2); the second
    call writes its final state over its own initial state (S_final aliases S0)."""
    T1, T2, H, d = 150, 90, 2, 128
    inp = inputs.prefill_inputs([T1 + T2], H, d, d, "bf16", s0_std=0.1, seed=5, device=DEV)
    o, S = run(inp)
    part = lambda s, e: {k: inp[k][s:e] for k in ("q", "k", "v", "log_alpha", "beta")}
    a = part(0, T1)
    cu1 = torch.tensor([0, T1], dtype=torch.int32, device=DEV)
    oa, Sa = kda_prefill(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], cu1, [0, T1],
                         S0=inp["S0"])
    b = part(T1, T1 + T2)
    cu2 = torch.tensor([0, T2], dtype=torch.int32, device=DEV)
    ob, Sb = kda_prefill(b["q"], b["k"], b["v"], b["log_alpha"], b["beta"], cu2, [0, T2],
                         S0=Sa, S_final=Sa)
    assert Sb.data_ptr() == Sa.data_ptr()
    # both runs carry the path's own rounding (fp16 tensor-core operands), so they
    # agree to twice the parity bound rather than bit for bit
    assert rel_l2(host64(torch.cat([oa, ob])), host64(o)) < 2 * TOL["bf16"]["o"]
    assert rel_l2(host64(Sb), host64(S)) < 2 * TOL["bf16"]["S"]
    compare_full(inp, o, S, "bf16")


def test_prefill_then_decode_equals_longer_prefill():
    T, n, H, d = 130, 4, 2, 128
    inp = inputs.prefill_inputs([T + n], H, d, d, "bf16", s0_std=0.1, seed=6, device=DEV)
    o_all, S_all = run(inp)
    cu = torch.tensor([0, T], dtype=torch.int32, device=DEV)
    sl = {k: inp[k][:T] for k in ("q", "k", "v", "log_alpha", "beta")}
    _, S = kda_prefill(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], cu, [0, T],
                       S0=inp["S0"])
    outs = []
    for t in range(T, T + n):
        outs.append(kda_decode_step(inp["q"][t:t + 1], inp["k"][t:t + 1], inp["v"][t:t + 1],
                                    inp["log_alpha"][t:t + 1], inp["beta"][t:t + 1], S))
    assert rel_l2(host64(torch.cat(outs)), host64(o_all[T:])) < 2 * TOL["bf16"]["o"]
    assert rel_l2(host64(S[0]), host64(S_all[0])) < 2 * TOL["bf16"]["S"]


def test_empty_sequences_keep_initial_state():
    inp = inputs.prefill_inputs([0, 5, 0], 2, 128, 128, "bf16", s0_std=0.1, seed=8, device=DEV)
    o, S = run(inp)
    torch.testing.assert_close(S[0], inp["S0"][0], rtol=0, atol=0)
    torch.testing.assert_close(S[2], inp["S0"][2], rtol=0, atol=0)
    compare_full(inp, o, S, "bf16")
    inp0 = inputs.prefill_inputs([0, 0], 1, 16, 16, "f32", s0_std=0.0, seed=8, device=DEV)
    o0, S0 = run(inp0, S0=None)
    assert o0.numel() == 0 and float(S0.abs().max()) == 0.0


def test_batched_prefill_workload_sampled():
    """8 x 8192 tokens, H = 32, d = 128, bf16: sampled (sequence, head) pairs."""
    w = inputs.WORKLOADS["batched_prefill"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, S = run(inp, chunk=w.chunk)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    units = [(0, 0), (7, 31), (3, 17), (5, 2)]
    compare_units(inp, o, S, units, "bf16")
    compare_heads(inp, o, S, [0, 13, 31], "bf16")


def test_longctx_varlen_workload_sampled():
    """1,048,576 packed tokens (one 524,288-token sequence + 64 shorter ones), H = 32,
    d = 128, bf16, in the launch configuration the bench times (the long sequence split
    into segments): every sequence on heads 0, 13 and 31 against the oracle, as one
    tensor per head subset."""
    w = inputs.WORKLOADS["longctx_varlen_prefill"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, S = run(inp, chunk=w.chunk)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    compare_heads(inp, o, S, [0, 13, 31], "bf16")


def test_long_sequence_last_is_scheduled_the_same():
    """Results do not depend on where the long sequence sits in the packing."""
    lens = [40, 33, 700]
    inp = inputs.prefill_inputs(lens, 2, 128, 128, "bf16", s0_std=0.1, seed=9, device=DEV)
    o, S = run(inp)
    compare_full(inp, o, S, "bf16")
