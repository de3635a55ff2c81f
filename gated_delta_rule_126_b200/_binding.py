"""ctypes binding of ``include/kda.h`` (argument marshalling only).

Every step of the operator runs in the CUDA library ``lib/libkda_b200.so``; this
module only turns torch tensors into pointers and sizes, allocates outputs with
torch when the caller does not pass them, and raises on a non-OK status.  There is
no CPU fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libkda_b200.so")

KDA_OK = 0
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_WORKSPACE", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_DEVICE_FAULT"}
DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1}

_lock = threading.Lock()
_lib = None


class KdaError(RuntimeError):
    """A KDA library call returned a status other than KDA_OK."""

    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__(f"{what}: {STATUS_NAMES.get(self.status, self.status)}")


def _declare(lib):
    c = ctypes
    vp, i32, i64, sz = c.c_void_p, c.c_int, c.c_int64, c.c_size_t
    lib.kda_status_string.restype = c.c_char_p
    lib.kda_status_string.argtypes = [i32]
    lib.kda_version.restype = i32
    lib.kda_version.argtypes = []
    lib.kda_prefill_workspace_size.restype = sz
    lib.kda_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
    lib.kda_prefill.restype = i32
    lib.kda_prefill.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                vp, vp, vp, sz, vp]
    lib.kda_prefill_gated.restype = i32
    lib.kda_prefill_gated.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                      vp, vp, c.c_float, vp, vp, vp, sz, vp]
    lib.kda_prologue.restype = i32
    lib.kda_prologue.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                 c.c_float, vp, vp, vp, vp, vp, vp]
    lib.kda_decode_step.restype = i32
    lib.kda_decode_step.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, vp]
    lib.kda_decode_tokens.restype = i32
    lib.kda_decode_tokens.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                      vp, vp]
    lib.kda_workspace_status.restype = i32
    lib.kda_workspace_status.argtypes = [vp, vp]
    lib.kda_backward_workspace_size.restype = sz
    lib.kda_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32]
    lib.kda_backward.restype = i32
    lib.kda_backward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp,
                                 vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_wait_timeout_selftest.restype = i32
    lib.kda_wait_timeout_selftest.argtypes = [vp, sz, c.c_longlong, vp]
    return lib


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"KDA CUDA library not found at {path}; build it with "
                    "`python -m gated_delta_rule_126_b200.build`")
            _lib = _declare(ctypes.CDLL(path))
    return _lib


def _check(status: int, what: str):
    if status != KDA_OK:
        raise KdaError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _dims(t, name, ndim):
    """Shape of t, which must be a tensor with ndim dimensions."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _shapes(**named):
    """Checks name=(tensor or None, expected shape) before any pointer reaches the library:
    the kernels trust the sizes they are given."""
    for name, (t, shape) in named.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _offsets(cu_seqlens, cu_seqlens_host, T):
    """(N, host copy of the offsets); the offsets must end within the T rows given.

    ``cu_seqlens_host`` must hold the same values as the device tensor ``cu_seqlens``:
    the host copy sizes the launches and is the one checked here, while the kernels
    read the device copy.  Offsets on the device that differ from the host copy (or
    end past the T rows) make the kernels read and write outside the tensors.  When
    in doubt, pass ``cu_seqlens_host=None``: the offsets are then copied from the
    device (which synchronises)."""
    if not isinstance(cu_seqlens, torch.Tensor) or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D tensor")
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu()
    cu_h = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    N = cu_h.numel() - 1
    if N < 0 or cu_seqlens.numel() != N + 1:
        raise ValueError("cu_seqlens and cu_seqlens_host differ in length")
    if int(cu_h[-1]) > T:
        raise ValueError(f"cu_seqlens ends at token {int(cu_h[-1])} but the inputs hold {T} tokens")
    return N, cu_h


def prefill_workspace_size(num_seqs, total_tokens, H, d_k, d_v, chunk=64, dtype=torch.bfloat16):
    return int(load().kda_prefill_workspace_size(int(num_seqs), int(total_tokens), int(H),
                                                 int(d_k), int(d_v), int(chunk),
                                                 DTYPE_CODE[dtype]))


def kda_prefill(q, k, v, log_alpha, beta, cu_seqlens, cu_seqlens_host=None, S0=None,
                chunk=64, o=None, S_final=None, workspace=None, stream=None):
    """Chunked KDA prefill over packed sequences (see ``kda_prefill`` in kda.h).

    q, k [T,H,d_k], v [T,H,d_v] (float32 or bfloat16), log_alpha [T,H,d_k] f32,
    beta [T,H] f32, cu_seqlens [N+1] int32 on the device, cu_seqlens_host the same
    offsets as a list or CPU tensor (copied from the device when omitted, which
    synchronises), S0 [N,H,d_k,d_v] f32 or None.  Returns ``(o, S_final)``.
    """
    lib = load()
    T, H, dk = _dims(q, "q", 3)
    dv = _dims(v, "v", 3)[2]
    N, cu_h = _offsets(cu_seqlens, cu_seqlens_host, T)
    _shapes(k=(k, (T, H, dk)), v=(v, (T, H, dv)), log_alpha=(log_alpha, (T, H, dk)), beta=(beta, (T, H)),
            S0=(S0, (N, H, dk, dv)), o=(o, (T, H, dv)), S_final=(S_final, (N, H, dk, dv)))
    dev = q.device
    dt = q.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("q/k/v dtype must be float32 or bfloat16")
    _need(q, "q", dt)
    _need(k, "k", dt, dev)
    _need(v, "v", dt, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
    if o is None:
        o = torch.empty(T, H, dv, dtype=dt, device=dev)
    if S_final is None:
        S_final = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    _need(o, "o", dt, dev)
    _need(S_final, "S_final", torch.float32, dev)
    ws_bytes = prefill_workspace_size(N, T, H, dk, dv, chunk, dt)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib.kda_prefill(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODE[dt], _ptr(log_alpha),
                             _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                             ctypes.c_void_p(cu_h.data_ptr()), N, H, dk, dv, int(chunk),
                             _ptr(o), _ptr(S_final), _ptr(workspace),
                             workspace.numel() * workspace.element_size(),
                             _stream_handle(stream))
    _check(st, "kda_prefill")
    return o, S_final


def kda_prefill_gated(q, k, v, log_alpha, beta, cu_seqlens, gate, norm_weight, eps=1e-6,
                      cu_seqlens_host=None, S0=None, chunk=64, y=None, S_final=None, workspace=None,
                      stream=None):
    """Chunked prefill with the output epilogue (see ``kda_prefill_gated`` in kda.h).

    As ``kda_prefill``, plus gate [T,H,d_v] (dtype of q), norm_weight [d_v] float32 and
    eps > 0; returns ``(y, S_final)`` with y = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate).
    """
    lib = load()
    T, H, dk = _dims(q, "q", 3)
    dv = _dims(v, "v", 3)[2]
    N, cu_h = _offsets(cu_seqlens, cu_seqlens_host, T)
    _shapes(k=(k, (T, H, dk)), v=(v, (T, H, dv)), log_alpha=(log_alpha, (T, H, dk)), beta=(beta, (T, H)),
            gate=(gate, (T, H, dv)), norm_weight=(norm_weight, (dv,)), S0=(S0, (N, H, dk, dv)),
            y=(y, (T, H, dv)), S_final=(S_final, (N, H, dk, dv)))
    dev = q.device
    dt = q.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("q/k/v dtype must be float32 or bfloat16")
    _need(q, "q", dt)
    _need(k, "k", dt, dev)
    _need(v, "v", dt, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(gate, "gate", dt, dev)
    _need(norm_weight, "norm_weight", torch.float32, dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
    if y is None:
        y = torch.empty(T, H, dv, dtype=dt, device=dev)
    if S_final is None:
        S_final = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    _need(y, "y", dt, dev)
    _need(S_final, "S_final", torch.float32, dev)
    ws_bytes = prefill_workspace_size(N, T, H, dk, dv, chunk, dt)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib.kda_prefill_gated(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODE[dt], _ptr(log_alpha),
                                   _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
                                   ctypes.c_void_p(cu_h.data_ptr()), N, H, dk, dv, int(chunk),
                                   _ptr(gate), _ptr(norm_weight), float(eps), _ptr(y),
                                   _ptr(S_final), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream))
    _check(st, "kda_prefill_gated")
    return y, S_final


def kda_prologue(q_pre, k_pre, v_pre, conv_q, conv_k, conv_v, a_gate, rate, b_gate, cu_seqlens,
                 cu_seqlens_host=None, l2_eps=1e-6, out=None, stream=None):
    """The layer's input prologue (see ``kda_prologue`` in kda.h).

    q_pre, k_pre [T,H,d_k], v_pre [T,H,d_v] (float32 or bfloat16); conv_* [H,d,W] float32;
    a_gate [T,H,d_k], rate [H], b_gate [T,H] float32.  Returns a dict with q, k, v,
    log_alpha, beta in kda_prefill's layouts (``out`` may supply them).
    """
    lib = load()
    T, H, dk = _dims(q_pre, "q_pre", 3)
    dv = _dims(v_pre, "v_pre", 3)[2]
    W = _dims(conv_q, "conv_q", 3)[2]
    N, cu_h = _offsets(cu_seqlens, cu_seqlens_host, T)
    given = dict(out or {})
    _shapes(k_pre=(k_pre, (T, H, dk)), v_pre=(v_pre, (T, H, dv)), conv_q=(conv_q, (H, dk, W)),
            conv_k=(conv_k, (H, dk, W)), conv_v=(conv_v, (H, dv, W)), a_gate=(a_gate, (T, H, dk)),
            rate=(rate, (H,)), b_gate=(b_gate, (T, H)), q=(given.get("q"), (T, H, dk)),
            k=(given.get("k"), (T, H, dk)), v=(given.get("v"), (T, H, dv)),
            log_alpha=(given.get("log_alpha"), (T, H, dk)), beta=(given.get("beta"), (T, H)))
    dev = q_pre.device
    dt = q_pre.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("projection dtype must be float32 or bfloat16")
    _need(q_pre, "q_pre", dt)
    _need(k_pre, "k_pre", dt, dev)
    _need(v_pre, "v_pre", dt, dev)
    for name, t in (("conv_q", conv_q), ("conv_k", conv_k), ("conv_v", conv_v), ("a_gate", a_gate),
                    ("rate", rate), ("b_gate", b_gate)):
        _need(t, name, torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    out = given
    out.setdefault("q", torch.empty(T, H, dk, dtype=dt, device=dev))
    out.setdefault("k", torch.empty(T, H, dk, dtype=dt, device=dev))
    out.setdefault("v", torch.empty(T, H, dv, dtype=dt, device=dev))
    out.setdefault("log_alpha", torch.empty(T, H, dk, dtype=torch.float32, device=dev))
    out.setdefault("beta", torch.empty(T, H, dtype=torch.float32, device=dev))
    for name in ("q", "k", "v"):
        _need(out[name], name, dt, dev)
    _need(out["log_alpha"], "log_alpha", torch.float32, dev)
    _need(out["beta"], "beta", torch.float32, dev)
    with torch.cuda.device(dev):
        st = lib.kda_prologue(_ptr(q_pre), _ptr(k_pre), _ptr(v_pre), DTYPE_CODE[dt], _ptr(conv_q),
                              _ptr(conv_k), _ptr(conv_v), int(W), _ptr(a_gate), _ptr(rate),
                              _ptr(b_gate), _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), N,
                              H, dk, dv, float(l2_eps), _ptr(out["q"]), _ptr(out["k"]),
                              _ptr(out["v"]), _ptr(out["log_alpha"]), _ptr(out["beta"]),
                              _stream_handle(stream))
    _check(st, "kda_prologue")
    return out


def kda_decode_step(q, k, v, log_alpha, beta, S, o=None, stream=None):
    """One decode step for B sequences (see ``kda_decode_step`` in kda.h).

    q, k [B,H,d_k], v [B,H,d_v], log_alpha [B,H,d_k] f32, beta [B,H] f32,
    S [B,H,d_k,d_v] f32 (updated in place).  Returns o [B,H,d_v].
    """
    lib = load()
    B, H, dk = _dims(q, "q", 3)
    dv = _dims(v, "v", 3)[2]
    _shapes(k=(k, (B, H, dk)), v=(v, (B, H, dv)), log_alpha=(log_alpha, (B, H, dk)), beta=(beta, (B, H)),
            S=(S, (B, H, dk, dv)), o=(o, (B, H, dv)))
    dev = q.device
    dt = q.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("q/k/v dtype must be float32 or bfloat16")
    _need(q, "q", dt)
    _need(k, "k", dt, dev)
    _need(v, "v", dt, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, dv, dtype=dt, device=dev)
    _need(o, "o", dt, dev)
    with torch.cuda.device(dev):
        st = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODE[dt], _ptr(log_alpha),
                                 _ptr(beta), _ptr(S), B, H, dk, dv, _ptr(o),
                                 _stream_handle(stream))
    _check(st, "kda_decode_step")
    return o


def kda_decode_tokens(q, k, v, log_alpha, beta, S_pool, slot_idx=None, o=None, stream=None):
    """n tokens for B sequences with states in a slot pool (see ``kda_decode_tokens`` in kda.h).

    q, k [B,n,H,d_k], v [B,n,H,d_v], log_alpha [B,n,H,d_k] f32, beta [B,n,H] f32,
    S_pool [num_slots,H,d_k,d_v] f32 (updated in place), slot_idx [B] int32 on the
    device or None (slot b).  Returns o [B,n,H,d_v].
    """
    lib = load()
    B, n, H, dk = _dims(q, "q", 4)
    dv = _dims(v, "v", 4)[3]
    ns = _dims(S_pool, "S_pool", 4)[0]
    _shapes(k=(k, (B, n, H, dk)), v=(v, (B, n, H, dv)), log_alpha=(log_alpha, (B, n, H, dk)),
            beta=(beta, (B, n, H)), S_pool=(S_pool, (ns, H, dk, dv)), slot_idx=(slot_idx, (B,)),
            o=(o, (B, n, H, dv)))
    dev = q.device
    dt = q.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("q/k/v dtype must be float32 or bfloat16")
    _need(q, "q", dt)
    _need(k, "k", dt, dev)
    _need(v, "v", dt, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S_pool, "S_pool", torch.float32, dev)
    if slot_idx is not None:
        _need(slot_idx, "slot_idx", torch.int32, dev)
    if o is None:
        o = torch.empty(B, n, H, dv, dtype=dt, device=dev)
    _need(o, "o", dt, dev)
    with torch.cuda.device(dev):
        st = lib.kda_decode_tokens(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODE[dt], _ptr(log_alpha),
                                   _ptr(beta), _ptr(S_pool), _ptr(slot_idx), S_pool.shape[0], B,
                                   n, H, dk, dv, _ptr(o), _stream_handle(stream))
    _check(st, "kda_decode_tokens")
    return o


def backward_workspace_size(num_seqs, total_tokens, H, d_k, d_v):
    return int(load().kda_backward_workspace_size(int(num_seqs), int(total_tokens), int(H), int(d_k),
                                                  int(d_v)))


def kda_backward(q, k, v, log_alpha, beta, cu_seqlens, dO, cu_seqlens_host=None, S0=None,
                 dS_final=None, want_dS0=True, workspace=None, stream=None):
    """Gradients of the KDA recurrence (see ``kda_backward`` in kda.h).

    Inputs as ``kda_prefill`` plus dO [T,H,d_v] (dtype of q) and dS_final
    [N,H,d_k,d_v] f32 or None.  Returns a dict of float32 tensors dq, dk, dv,
    dlog_alpha, dbeta and dS0 (None unless ``want_dS0``).  dq, dk, dlog_alpha and
    dbeta are added up from 16-channel slices with float32 atomics, so repeated
    calls can differ in their last bits; dv and dS0 do not.
    """
    lib = load()
    T, H, dk = _dims(q, "q", 3)
    dv = _dims(v, "v", 3)[2]
    N, cu_h = _offsets(cu_seqlens, cu_seqlens_host, T)
    _shapes(k=(k, (T, H, dk)), v=(v, (T, H, dv)), dO=(dO, (T, H, dv)), log_alpha=(log_alpha, (T, H, dk)),
            beta=(beta, (T, H)), S0=(S0, (N, H, dk, dv)), dS_final=(dS_final, (N, H, dk, dv)))
    dev = q.device
    dt = q.dtype
    if dt not in DTYPE_CODE:
        raise ValueError("q/k/v dtype must be float32 or bfloat16")
    _need(q, "q", dt)
    _need(k, "k", dt, dev)
    _need(v, "v", dt, dev)
    _need(dO, "dO", dt, dev)
    _need(log_alpha, "log_alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    for t, name in ((S0, "S0"), (dS_final, "dS_final")):
        if t is not None:
            _need(t, name, torch.float32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty(T, H, dk, **f32), dk=torch.empty(T, H, dk, **f32),
               dv=torch.empty(T, H, dv, **f32), dlog_alpha=torch.empty(T, H, dk, **f32),
               dbeta=torch.empty(T, H, **f32),
               dS0=torch.empty(N, H, dk, dv, **f32) if want_dS0 else None)
    ws_bytes = backward_workspace_size(N, T, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), DTYPE_CODE[dt], _ptr(log_alpha), _ptr(beta),
                              _ptr(S0), _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), N, H, dk, dv,
                              _ptr(dO), _ptr(dS_final), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                              _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]), _ptr(out["dS0"]),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream_handle(stream))
    _check(st, "kda_backward")
    return out

def workspace_status(workspace, stream=None):
    """Status flagged by the kernels of the last prefill that used ``workspace``."""
    return int(load().kda_workspace_status(_ptr(workspace), _stream_handle(stream)))


def wait_timeout_selftest(workspace, max_cycles, stream=None):
    """Run the kernel whose bounded waits never see their event (see
    ``kda_wait_timeout_selftest`` in kda.h); the caller reads the flag it leaves
    with :func:`workspace_status`."""
    _need(workspace, "workspace", torch.uint8)
    st = load().kda_wait_timeout_selftest(_ptr(workspace), workspace.numel(), int(max_cycles),
                                          _stream_handle(stream))
    _check(st, "kda_wait_timeout_selftest")
