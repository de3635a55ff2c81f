"""Parity over the whole decay range alpha in [0, 1] (needs a GPU).

The wiki page "Kimi Linear 高效注意力架构" (section "Kimi Delta Attention (KDA)",
"Channel-wise 衰减" bullet) allows any per-channel decay alpha in [0, 1]^{d_k}; the
workloads' recipe (-0.1 softplus) only covers mild decays.  These tests drive the
chunked paths (tensor-core bf16 and CUDA-core fp32, plain and gated, unsplit and
split) and both decode kernels with strong decays (log alpha = -c softplus(N(0, 1)),
c = 1, 4, 16), fast- and slow-forgetting channels in one head, and channels erased
outright (log alpha = -inf, alpha = 0), and hold them to the same bounds as every
other parity test.  No output may be NaN or infinite.
"""
import pytest
import torch

import oracle
from oracle import epilogue
from gated_delta_rule_126_b200 import (inputs, kda_backward, kda_decode_step, kda_decode_tokens,
                                       kda_prefill, kda_prefill_gated)
from tests.kda_check import TOL, compare_full, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENS = [1, 17, 64, 65, 0, 130, 3, 200]


def _inp(lens, H, dk, dv, dtype, scale, zero_frac=0.0, seed=61):
    inp = inputs.prefill_inputs(lens, H, dk, dv, dtype, s0_std=0.1, seed=seed, device=DEV)
    inp["log_alpha"] = inputs.decay_log_alpha(sum(lens), H, dk, scale, zero_frac, seed=seed + 100, device=DEV)
    return inp


def _mixed_scale(dk):
    # even channels forget slowly (the workloads' rate), odd channels fast
    sc = torch.full((dk,), 0.1)
    sc[1::2] = 16.0
    return sc


def _prefill(inp, chunk=64, **kw):
    o, S = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"],
                       inp["cu_seqlens_host"], S0=inp["S0"], chunk=chunk, **kw)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    return o, S


@pytest.mark.parametrize("scale", [1.0, 4.0, 16.0, "mixed"])
@pytest.mark.parametrize("zero_frac", [0.0, 0.02])
def test_tensor_core_strong_decay(scale, zero_frac):
    """bf16 q/k/v, d = 128, chunk 64: the tensor-core path, ragged packing."""
    sc = _mixed_scale(128) if scale == "mixed" else scale
    inp = _inp(LENS, 3, 128, 128, "bf16", sc, zero_frac)
    o, S = _prefill(inp)
    compare_full(inp, o, S, "bf16")


@pytest.mark.parametrize("scale", [1.0, 4.0, 16.0, "mixed"])
@pytest.mark.parametrize("dk,dv,chunk", [(128, 128, 64), (32, 48, 16), (64, 64, 32)])
def test_fp32_strong_decay(scale, dk, dv, chunk):
    """float32 q/k/v: the CUDA-core chunk path at the 1e-5 bound, with 2% erased channels."""
    sc = _mixed_scale(dk) if scale == "mixed" else scale
    inp = _inp(LENS, 2, dk, dv, "f32", sc, 0.02)
    o, S = _prefill(inp, chunk=chunk)
    compare_full(inp, o, S, "f32")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_whole_tokens_erased(dtype):
    """Every channel of some tokens has alpha = 0, at a chunk's first, middle and last
    token and in a partial chunk: the state restarts there."""
    lens = [150, 64, 70]
    inp = _inp(lens, 2, 128, 128, dtype, 1.0)
    for t in (0, 31, 63, 64, 100, 149, 150, 214, 283):
        inp["log_alpha"][t] = float("-inf")
    o, S = _prefill(inp)
    compare_full(inp, o, S, dtype)


def test_gated_prefill_strong_decay():
    """The fused output epilogue on strong decays with erased channels."""
    inp = _inp(LENS, 2, 128, 128, "bf16", 4.0, 0.02)
    gate, w = inputs.gate_inputs(sum(LENS), 2, 128, "bf16", seed=62, device=DEV)
    y, S = kda_prefill_gated(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"],
                             gate, w, 1e-6, cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"])
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all() and torch.isfinite(S).all()
    o_ref, S_ref = oracle.prefill(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), host64(inp["log_alpha"]),
                                  host64(inp["beta"]), inp["cu_seqlens_host"], S0=host64(inp["S0"]))
    y_ref = epilogue.gated_rmsnorm(o_ref, host64(gate), host64(w), 1e-6)
    assert rel_l2(host64(y), y_ref) <= TOL["bf16"]["o"]
    assert rel_l2(host64(S), S_ref) <= TOL["bf16"]["S"]


@pytest.mark.parametrize("scale", [1.0, "mixed"])
def test_split_path_strong_decay(scale):
    """A 20,000-token sequence (split into segments on the tensor-core path: the segment
    transitions compose strong decays and erased channels) next to a short one."""
    sc = _mixed_scale(128) if scale == "mixed" else scale
    inp = _inp([20000, 300], 1, 128, 128, "bf16", sc, 0.01)
    o, S = _prefill(inp)
    compare_full(inp, o, S, "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("scale,zero_frac", [(4.0, 0.02), (2.0, 0.0), (1.0, 0.0)])
def test_decode_strong_decay(dtype, scale, zero_frac):
    """Single-step and multi-token decode with strong decays and erased channels, at three
    decay rates.  Nine tokens make two full staged groups of four and a single token in
    the multi-token kernel."""
    B, H, d, n = 6, 2, 128, 9
    dinp = inputs.decode_inputs(B, H, d, d, n, dtype, seed=63, device=DEV)
    dinp["log_alpha"] = inputs.decay_log_alpha(n * B, H, d, scale, zero_frac, seed=64,
                                               device=DEV).reshape(n, B, H, d)
    S = dinp["S0"].clone()
    outs = [kda_decode_step(dinp["q"][t], dinp["k"][t], dinp["v"][t], dinp["log_alpha"][t], dinp["beta"][t], S)
            for t in range(n)]
    tok = lambda x: x.transpose(0, 1).contiguous()  # [n, B, ...] -> [B, n, ...]
    pool = dinp["S0"].clone()
    o_tok = kda_decode_tokens(tok(dinp["q"]), tok(dinp["k"]), tok(dinp["v"]), tok(dinp["log_alpha"]),
                              tok(dinp["beta"]), pool)
    torch.cuda.synchronize()
    o_step = torch.stack(outs)  # [n, B, H, d]
    for b in range(B):
        sl = lambda x: host64(x[:, b])
        o_ref, S_ref = oracle.prefill(sl(dinp["q"]), sl(dinp["k"]), sl(dinp["v"]), sl(dinp["log_alpha"]),
                                      sl(dinp["beta"]), [0, n], S0=host64(dinp["S0"][b:b + 1]))
        tol = TOL[dtype]
        assert rel_l2(host64(o_step[:, b]), o_ref) <= tol["o"]
        assert rel_l2(host64(S[b]), S_ref[0]) <= tol["S"]
        assert rel_l2(host64(o_tok[b]), o_ref) <= tol["o"]
        assert rel_l2(host64(pool[b]), S_ref[0]) <= tol["S"]


def test_backward_strong_decay():
    """The backward pass's gradients with strong decays and erased channels, at the
    backward's 1e-5 bound (the gradient of an erased channel's log alpha is zero)."""
    lens = [70, 1, 33]
    inp = _inp(lens, 2, 64, 48, "f32", 4.0, 0.02)
    dO, dS = inputs.grad_inputs(sum(lens), len(lens), 2, 64, 48, "f32", seed=65, device=DEV)
    g = kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"], dO,
                     cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"], dS_final=dS)
    torch.cuda.synchronize()
    ref = oracle.backward(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]), host64(inp["log_alpha"]),
                          host64(inp["beta"]), inp["cu_seqlens_host"], host64(dO), S0=host64(inp["S0"]),
                          dS_final=host64(dS))
    for name, r in ref.items():
        assert torch.isfinite(g[name]).all(), name
        assert rel_l2(host64(g[name]), r) <= 1e-5, name


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mild_and_strong_chunks_alternate(dtype):
    """Decay strength changes along the sequence (mild 64-token stretches between strong
    ones, erased channels only in the strong ones): the tensor-core path switches its
    factoring from chunk to chunk and must carry the state across every switch."""
    lens = [64 * 7 - 9, 150]
    T = sum(lens)
    per_tok = torch.tensor(([0.1] * 64 + [4.0] * 64 + [0.1] * 128 + [16.0] * 64 + [0.1] * 64 + [1.0] * 64)[:lens[0]]
                           + [0.1] * 70 + [4.0] * 80, dtype=torch.float32)
    inp = _inp(lens, 2, 128, 128, dtype, 1.0)
    la = inputs.decay_log_alpha(T, 2, 128, per_tok.view(T, 1, 1).to(DEV), 0.0, seed=66, device=DEV)
    zeros = inputs.decay_log_alpha(T, 2, 128, 1.0, 0.02, seed=67, device=DEV)
    strong = (per_tok > 0.5).view(T, 1, 1).to(DEV)
    inp["log_alpha"] = torch.where(strong & torch.isinf(zeros), zeros, la).contiguous()
    o, S = _prefill(inp)
    compare_full(inp, o, S, dtype)
