"""The C-ABI library loads, exports every symbol kda.h declares, and rejects bad
arguments on the host (no GPU needed: every check here returns before any CUDA
call is made)."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_126_b200 import _binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _binding.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    assert declared_symbols() == sorted([
        "kda_backward", "kda_backward_workspace_size", "kda_decode_step", "kda_decode_tokens", "kda_prefill", "kda_prefill_gated", "kda_prefill_noalloc", "kda_prologue",
        "kda_prefill_workspace_size", "kda_status_string", "kda_version", "kda_wait_timeout_selftest",
        "kda_workspace_status"])


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # nothing else is exported from the library's own code
    out = os.popen(f"nm -D --defined-only {_binding.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and "kda" in ln}
    assert exported == set(declared_symbols())


def test_status_strings_and_version(lib):
    for code, name in _binding.STATUS_NAMES.items():
        assert lib.kda_status_string(code).decode() == name
    assert lib.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"
    assert lib.kda_version() >= 100


def test_workspace_size(lib):
    ws = lib.kda_prefill_workspace_size
    assert ws(8, 65536, 32, 128, 128, 64, 1) >= 256
    assert ws(8, 65536, 32, 128, 128, 48, 1) == 0        # unsupported chunk
    assert ws(8, 65536, 32, 129, 128, 64, 1) == 0        # d_k too large
    assert ws(-1, 0, 32, 128, 128, 64, 1) == 0
    assert ws(1, -5, 32, 128, 128, 64, 1) == 0
    assert ws(1, 1 << 40, 32, 128, 128, 64, 1) == 0      # more tokens than int32 offsets
    # the tensor-core shapes reserve room for the sequence split once a call can hold one
    # (at least 16,384 tokens): three [slot][H][128][128] float32 arrays
    small, big = ws(2, 8192, 32, 128, 128, 64, 1), ws(2, 1 << 20, 32, 128, 128, 64, 1)
    assert small < 4096 and big >= 3 * 3 * 3 * 32 * 128 * 128 * 4
    assert ws(2, 1 << 20, 32, 64, 64, 64, 1) < 4096      # CUDA-core path: no split


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every case fails on the host


def _prefill(lib, cu_host, N, H=2, dk=16, dv=16, chunk=16, dtype=0, ptr=FAKE, ws=FAKE,
             ws_bytes=1 << 20, s0=None, out=FAKE):
    arr = (ctypes.c_int32 * len(cu_host))(*cu_host) if cu_host is not None else None
    return lib.kda_prefill(ptr, ptr, ptr, dtype, ptr, ptr, s0, FAKE, arr, N, H, dk, dv, chunk,
                           out, out, ws, ws_bytes, None)


def test_prefill_rejects_bad_arguments(lib):
    assert _prefill(lib, [0, 4], 1, H=0) == INVALID
    assert _prefill(lib, [0, 4], 1, dk=0) == INVALID
    assert _prefill(lib, [0, 4], 1, dtype=7) == INVALID
    assert _prefill(lib, [0, 4], -1) == INVALID
    assert _prefill(lib, [0, 4], 1, chunk=48) == UNSUPPORTED
    assert _prefill(lib, [0, 4], 1, dk=256) == UNSUPPORTED
    assert _prefill(lib, None, 1) == INVALID                     # no host offsets
    assert _prefill(lib, [1, 4], 1) == INVALID                   # must start at 0
    assert _prefill(lib, [0, 4, 3], 2) == INVALID                # decreasing
    assert _prefill(lib, [0, 4], 1, ptr=None) == INVALID         # null inputs
    assert _prefill(lib, [0, 4], 1, ptr=ctypes.c_void_p((1 << 20) + 4)) == INVALID  # misaligned
    assert _prefill(lib, [0, 4], 1, out=None) == INVALID         # null outputs
    assert _prefill(lib, [0, 4], 1, s0=ctypes.c_void_p((1 << 20) + 8)) == INVALID
    assert _prefill(lib, [0, 4], 1, ws=None) == WORKSPACE
    assert _prefill(lib, [0, 4], 1, ws_bytes=16) == WORKSPACE
    assert _prefill(lib, [0, 4], 1, ws=ctypes.c_void_p((1 << 20) + 64)) == WORKSPACE


def _gated(lib, cu_host, N, H=2, dk=128, dv=128, chunk=64, dtype=1, gate=FAKE, w=FAKE, eps=1e-6,
           ws=FAKE):
    arr = (ctypes.c_int32 * len(cu_host))(*cu_host)
    return lib.kda_prefill_gated(FAKE, FAKE, FAKE, dtype, FAKE, FAKE, None, FAKE, arr, N, H, dk, dv,
                                 chunk, gate, w, eps, FAKE, FAKE, ws, 1 << 20, None)


def test_prefill_gated_rejects_bad_arguments(lib):
    assert _gated(lib, [0, 4], 1, H=0) == INVALID                  # kda_prefill's checks come first
    assert _gated(lib, [0, 4], 1, chunk=48) == UNSUPPORTED
    assert _gated(lib, [0, 4], 1, ws=None) == WORKSPACE
    assert _gated(lib, [0, 4], 1, eps=0.0) == INVALID
    assert _gated(lib, [0, 4], 1, eps=-1.0) == INVALID
    assert _gated(lib, [0, 4], 1, eps=float("inf")) == INVALID
    assert _gated(lib, [0, 4], 1, eps=float("nan")) == INVALID
    assert _gated(lib, [0, 4], 1, gate=None) == INVALID
    assert _gated(lib, [0, 4], 1, w=None) == INVALID
    assert _gated(lib, [0, 4], 1, gate=ctypes.c_void_p((1 << 20) + 4)) == INVALID  # misaligned
    assert _gated(lib, [0, 4], 1, dk=64, dv=64) == UNSUPPORTED    # bf16 off the fused path
    assert _gated(lib, [0, 4], 1, chunk=32) == UNSUPPORTED
    assert _gated(lib, [0], 0) == 0                                 # nothing to do


def _prologue(lib, cu_host, N, H=2, dk=128, dv=128, W=4, dtype=1, ptr=FAKE, eps=1e-6, q=FAKE):
    arr = (ctypes.c_int32 * len(cu_host))(*cu_host)
    return lib.kda_prologue(ptr, ptr, ptr, dtype, FAKE, FAKE, FAKE, W, FAKE, FAKE, FAKE, FAKE, arr, N, H, dk,
                            dv, eps, q, FAKE, FAKE, FAKE, FAKE, None)


def test_prologue_rejects_bad_arguments(lib):
    assert _prologue(lib, [0, 4], 1, H=0) == INVALID
    assert _prologue(lib, [0, 4], 1, dtype=5) == INVALID
    assert _prologue(lib, [0, 4], 1, eps=-1.0) == INVALID
    assert _prologue(lib, [0, 4], 1, eps=float("nan")) == INVALID
    assert _prologue(lib, [0, 4], 1, W=0) == UNSUPPORTED
    assert _prologue(lib, [0, 4], 1, W=5) == UNSUPPORTED
    assert _prologue(lib, [0, 4], 1, dk=130) == UNSUPPORTED
    assert _prologue(lib, [0, 4], 1, dv=126) == UNSUPPORTED
    assert _prologue(lib, [1, 4], 1) == INVALID                     # must start at 0
    assert _prologue(lib, [0, 4, 2], 2) == INVALID                  # decreasing
    assert _prologue(lib, [0, 4], 1, ptr=None) == INVALID
    assert _prologue(lib, [0, 4], 1, q=ctypes.c_void_p((1 << 20) + 8)) == INVALID  # misaligned
    assert _prologue(lib, [0, 0], 1) == 0                           # no tokens


def test_decode_rejects_bad_arguments(lib):
    f = lib.kda_decode_step
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, -1, 2, 128, 128, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, 4, 0, 128, 128, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, 4, 2, 128, 130, FAKE, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, 4, 2, 128, 126, FAKE, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, 4, 2, 128, 128, FAKE, None) == INVALID
    assert f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, ctypes.c_void_p((1 << 20) + 4), 4, 2, 128, 128,
             FAKE, None) == INVALID
    assert f(None, None, None, 1, None, None, None, 0, 2, 128, 128, None, None) == 0  # B = 0


def test_decode_tokens_rejects_bad_arguments(lib):
    f = lib.kda_decode_tokens
    args = lambda **kw: [kw.get("q", FAKE), FAKE, FAKE, kw.get("dt", 1), FAKE, FAKE, kw.get("S", FAKE),
                         kw.get("slots", FAKE), kw.get("ns", 8), kw.get("B", 4), kw.get("n", 2),
                         kw.get("H", 2), 128, kw.get("dv", 128), FAKE, None]
    assert f(*args(B=-1)) == INVALID
    assert f(*args(n=-1)) == INVALID
    assert f(*args(H=0)) == INVALID
    assert f(*args(ns=-1)) == INVALID
    assert f(*args(dt=3)) == INVALID
    assert f(*args(dv=126)) == UNSUPPORTED
    assert f(*args(slots=None, ns=2)) == INVALID          # identity slots need num_slots >= B
    assert f(*args(q=None)) == INVALID
    assert f(*args(S=ctypes.c_void_p((1 << 20) + 4))) == INVALID
    assert f(*args(n=0)) == 0 and f(*args(B=0)) == 0


def test_backward_workspace_size(lib):
    ws = lib.kda_backward_workspace_size
    n = ws(2, 16384, 32, 128, 128)
    # status + checkpoints (16384/32 + 3 blocks x 32 heads x 8 slices x 8 KiB) + w (16384 x 32 x 128 x 4)
    assert n == 256 + 515 * 32 * 8 * 8192 + 16384 * 32 * 128 * 4
    assert ws(1, 10, 1, 7, 5) > 256
    assert ws(1, 10, 1, 129, 5) == 0 and ws(1, 10, 1, 7, 129) == 0
    assert ws(-1, 10, 1, 7, 5) == 0 and ws(1, -1, 1, 7, 5) == 0 and ws(1, 10, 0, 7, 5) == 0
    assert ws(1, 1 << 40, 1, 7, 5) == 0


def _backward(lib, cu, N, dtype=1, H=2, dk=128, dv=128, ws_bytes=None, **kw):
    arr = (ctypes.c_int32 * len(cu))(*cu)
    ws = lib.kda_backward_workspace_size(N, cu[-1] if cu else 0, H, dk, dv) if ws_bytes is None else ws_bytes
    ptr = [kw.get(n, FAKE) for n in ("q", "k", "v")]
    return lib.kda_backward(*ptr, dtype, FAKE, FAKE, None, FAKE, arr, N, H, dk, dv, kw.get("dO", FAKE), None,
                            FAKE, FAKE, FAKE, FAKE, FAKE, None, kw.get("ws", FAKE), ws, None)


def test_backward_rejects_bad_arguments(lib):
    assert _backward(lib, [0, 4], 1, dtype=3) == INVALID
    assert _backward(lib, [0, 4], 1, H=0) == INVALID
    assert _backward(lib, [0, 4], 1, dk=129) == UNSUPPORTED
    assert _backward(lib, [0, 4], 1, dv=129) == UNSUPPORTED
    assert _backward(lib, [1, 4], 1) == INVALID                 # cu_seqlens[0] != 0
    assert _backward(lib, [0, 4, 2], 2) == INVALID              # decreasing offsets
    assert _backward(lib, [0, 4], 1, q=None) == INVALID
    assert _backward(lib, [0, 4], 1, dO=None) == INVALID
    assert _backward(lib, [0, 4], 1, ws=None) == WORKSPACE
    assert _backward(lib, [0, 4], 1, ws_bytes=256) == WORKSPACE
    assert _backward(lib, [0, 4], 1, ws=ctypes.c_void_p((1 << 20) + 16)) == WORKSPACE
    assert _backward(lib, [0], 0) == 0                          # no sequences: nothing to do
    assert _backward(lib, [0] * 65537, 65536, H=4096) == UNSUPPORTED  # grid of 2^31 blocks


def test_wait_timeout_selftest_rejects_bad_arguments(lib):
    f = lib.kda_wait_timeout_selftest
    assert f(None, 256, 1000, None) == WORKSPACE
    assert f(FAKE, 255, 1000, None) == WORKSPACE                      # shorter than the status block
    assert f(ctypes.c_void_p((1 << 20) + 16), 256, 1000, None) == WORKSPACE  # not 256-byte aligned
    assert f(FAKE, 256, 0, None) == INVALID
    assert f(FAKE, 256, 4000000001, None) == INVALID


def test_binding_raises_without_library(tmp_path):
    saved = _binding._lib
    try:
        _binding._lib = None
        with pytest.raises(RuntimeError, match="not found"):
            _binding.load(str(tmp_path / "missing.so"))
    finally:
        _binding._lib = saved


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure mode")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    # arguments pass the host checks, then the first CUDA call fails: KDA_ERR_CUDA, no crash
    assert _prefill(lib, [0, 4], 1) == 4
    assert _gated(lib, [0, 4], 1) == 4
    assert _gated(lib, [0, 4], 1, dtype=0, dk=16, dv=16, chunk=16) == 4
    assert _prologue(lib, [0, 4], 1) == 4
    assert _backward(lib, [0, 4], 1) == 4
