"""A bounded wait that runs out is reported, not hung on (needs a GPU).

Every spin inside the prefill kernels (on an mbarrier phase or on a shared-memory
progress counter) gives up after a fixed number of SM cycles, sets the status word
at the start of the workspace and returns.  kda_wait_timeout_selftest runs the same
two kinds of wait on events that nothing produces, with a short limit, so both run
out.  The test checks that the kernel ends in about the limit, that
kda_workspace_status reports KDA_ERR_DEVICE_FAULT (and clears the word), and that
the context is still usable: a prefill on the same workspace afterwards matches the
oracle and leaves the status clean.  No GPU fault, trap or hang is involved.
"""
import pytest
import torch

from gated_delta_rule_126_b200 import _binding, inputs, kda_prefill, prefill_workspace_size
from tests.kda_check import compare_full

pytestmark = pytest.mark.gpu
DEV = "cuda"
KDA_OK, KDA_ERR_DEVICE_FAULT = 0, 5
LIMIT_CYCLES = 200_000_000  # about 0.1 s at the B200's 1.965 GHz top SM clock


def _workspace(inp, chunk):
    T, H, dk = inp["q"].shape
    n = len(inp["cu_seqlens_host"]) - 1
    size = prefill_workspace_size(n, T, H, dk, inp["v"].shape[2], chunk, inp["q"].dtype)
    return torch.zeros(size, dtype=torch.uint8, device=DEV)


def test_wait_that_runs_out_sets_the_status_and_leaves_the_context_usable():
    w = inputs.WORKLOADS["tiny_f32"]
    inp = inputs.workload_inputs(w, device=DEV)
    ws = _workspace(inp, w.chunk)
    stream = torch.cuda.current_stream()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    _binding.wait_timeout_selftest(ws, LIMIT_CYCLES, stream)
    end.record(stream)
    end.synchronize()
    ms = start.elapsed_time(end)
    # the waits end by their limit: no faster than the top clock allows, far below a hang
    assert LIMIT_CYCLES / 2.2e9 * 1e3 <= ms < 5000.0, ms

    detail = int(ws[4:8].view(torch.int32).item())
    assert detail == 3, detail  # both the mbarrier wait and the counter wait ran out
    assert _binding.workspace_status(ws, stream) == KDA_ERR_DEVICE_FAULT
    assert _binding.workspace_status(ws, stream) == KDA_OK  # the flag was cleared

    o, S = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       inp["cu_seqlens"], inp["cu_seqlens_host"], S0=inp["S0"], chunk=w.chunk,
                       workspace=ws, stream=stream)
    assert _binding.workspace_status(ws, stream) == KDA_OK
    compare_full(inp, o, S, "f32")


def test_tensor_core_prefill_after_a_timeout():
    """The bf16 tensor-core kernel (TMEM, TMA) runs normally after the self-test."""
    w = inputs.WORKLOADS["single_seq_prefill"]
    inp = inputs.workload_inputs(w, device=DEV)
    ws = _workspace(inp, w.chunk)
    stream = torch.cuda.current_stream()
    _binding.wait_timeout_selftest(ws, LIMIT_CYCLES // 4, stream)
    assert _binding.workspace_status(ws, stream) == KDA_ERR_DEVICE_FAULT
    o, S = kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       inp["cu_seqlens"], inp["cu_seqlens_host"], S0=inp["S0"], chunk=w.chunk,
                       workspace=ws, stream=stream)
    assert _binding.workspace_status(ws, stream) == KDA_OK
    compare_full(inp, o, S, "bf16")
