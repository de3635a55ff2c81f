"""kda_prefill_noalloc against kda_prefill (needs a GPU).

kda_prefill_noalloc serves callers that cannot allocate device memory where they
run the operator (a host framework that owns every allocation, a plug-in handed
only its inputs and outputs).  It keeps its scratch in a device array inside the
library instead of a caller workspace.  This test calls it through the C ABI on
two calls in a row with different batches, so that scratch left by the first call
cannot leak into the second.  None of these batches is long enough for
kda_prefill's sequence split, so both entry points run the same kernels on the same
inputs: their outputs must be bit-identical (a scratch-reuse bug that shifts values
slightly would show here), and each batch is also held to the parity bounds against
the fp64 oracle.  The file name puts it last in collection order.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_126_b200 import _binding, inputs, kda_prefill
from tests.kda_check import compare_full

pytestmark = pytest.mark.gpu
DEV = "cuda"
KDA_ERR_WORKSPACE = 3
MAX_SEQS = 65536  # KDA_NOALLOC_MAX_SEQS in include/kda.h


def _lib():
    lib = _binding.load()
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.kda_prefill_noalloc.restype = i32
    lib.kda_prefill_noalloc.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                        i32, vp, vp, vp]
    return lib


def _noalloc(lib, inp, chunk):
    q = inp["q"]
    T, H, dk = q.shape
    dv = inp["v"].shape[2]
    N = len(inp["cu_seqlens_host"]) - 1
    o = torch.empty(T, H, dv, dtype=q.dtype, device=DEV)
    S = torch.empty(N, H, dk, dv, dtype=torch.float32, device=DEV)
    cu_h = torch.tensor(inp["cu_seqlens_host"], dtype=torch.int32)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.kda_prefill_noalloc(ptr(q), ptr(inp["k"]), ptr(inp["v"]), _binding.DTYPE_CODE[q.dtype],
                                 ptr(inp["log_alpha"]), ptr(inp["beta"]), ptr(inp["S0"]),
                                 ptr(inp["cu_seqlens"]), ctypes.c_void_p(cu_h.data_ptr()), N, H,
                                 dk, dv, chunk, ptr(o), ptr(S),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _binding.STATUS_NAMES.get(st, st)
    return o, S


@pytest.mark.parametrize("dtype,d,chunk", [("bf16", 128, 64), ("f32", 32, 16)])
def test_noalloc_matches_prefill_on_two_calls(dtype, d, chunk):
    lib = _lib()
    batches = [([300, 1, 64, 130], 2, 11), ([7, 513, 0, 64, 65, 200], 3, 12)]
    for lens, H, seed in batches:
        inp = inputs.prefill_inputs(lens, H, d, d, dtype, s0_std=0.1, seed=seed, device=DEV)
        o_ref, S_ref = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                   inp["cu_seqlens"], inp["cu_seqlens_host"], S0=inp["S0"],
                                   chunk=chunk)
        o, S = _noalloc(lib, inp, chunk)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), "o differs from kda_prefill's"
        assert torch.equal(S, S_ref), "S_final differs from kda_prefill's"
        compare_full(inp, o, S, dtype)


def test_noalloc_rejects_more_sequences_than_its_scratch_holds():
    lib = _lib()
    n = MAX_SEQS + 1
    cu = (ctypes.c_int32 * (n + 1))(*([0] * (n + 1)))
    fake = ctypes.c_void_p(1 << 20)
    st = lib.kda_prefill_noalloc(fake, fake, fake, 1, fake, fake, None, fake, cu, n, 1, 128, 128,
                                 64, fake, fake, None)
    assert st == KDA_ERR_WORKSPACE
