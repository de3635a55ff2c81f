"""fp64 CPU oracle for the Kimi Delta Attention (KDA) operator.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
imports, links or calls it, and it never imports the CUDA library: the two share
no code.  Inputs reach both sides from the seeded generators in
``gated_delta_rule_126_b200.inputs`` (which hold none of the method's arithmetic).

Contents
--------
* ``kda_oracle.c`` -- the token-by-token fp64 recurrence (the plain definition of
  the KDA state update from the wiki page "Kimi Linear 高效注意力架构", section
  "Kimi Delta Attention (KDA)", state-update equation, with the delta-rule
  read-out o_t = S_t^T q_t).  Compiled on demand with gcc into ``oracle/_build``.
* ``chunk_model.py`` -- the same operator rewritten chunk by chunk (WY/UT form)
  in fp64 numpy; it is pinned to the recurrence and gives per-stage values.
* ``kda_oracle_bwd.c`` -- the exact reverse-mode (adjoint) sweep of the same
  recurrence in fp64: gradients of <dO, o> + <dS_final, S_final> with respect to
  every input.  Pinned by central finite differences of the forward oracle
  (``tests/test_backward_pins.py``).
* ``epilogue.py`` / ``prologue.py`` -- the KDA layer's output epilogue and input
  prologue in fp64 numpy.

Parity status: the recurrence is pinned by the tests in
``tests/test_oracle_pins.py`` (closed forms, special cases, brute-force matrix
products, a hand-worked example) and ``tests/test_oracle_mutants.py`` (planted
mistakes must fail a pin).  The read-out o_t = S_t^T q_t is not printed on the
pages; it is pinned only by the delta-rule convention (post-update state), which
the exact-reconstruction and linear-attention pins exercise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libkda_oracle.so")
_BWD_SRC = os.path.join(_HERE, "kda_oracle_bwd.c")
_BWD_LIB_PATH = os.path.join(_BUILD, "libkda_oracle_bwd.so")
_lock = threading.Lock()
_lib = None
_bwd_lib = None

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-pthread", "-std=c99", "-Wall"]


def compile_c(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile an oracle C source into a shared library with gcc; return its path."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", *GCC_FLAGS, *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def build() -> str:
    """Build the oracle libraries if they are missing or older than their sources."""
    for src, out in ((_SRC, _LIB_PATH), (_BWD_SRC, _BWD_LIB_PATH)):
        if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
            compile_c(src, out)
    return _LIB_PATH


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kda_oracle_prefill.restype = ctypes.c_int
    lib.kda_oracle_prefill.argtypes = [dp, dp, dp, dp, dp, ctypes.c_void_p,
                                       ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       dp, dp, ctypes.c_int]
    lib.kda_oracle_default_threads.restype = ctypes.c_int
    lib.kda_oracle_default_threads.argtypes = []
    return lib


def load_library(path: str | None = None):
    """Load (building first if needed) the oracle shared library via ctypes."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def default_threads() -> int:
    return int(load_library().kda_oracle_default_threads())


def _f64(x, shape=None):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None:
        a = a.reshape(shape)
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def prefill(q, k, v, log_alpha, beta, cu_seqlens, S0=None, nthreads: int = 0, lib=None):
    """Run the fp64 recurrence over a packed batch of sequences.

    Shapes: q, k, log_alpha [T, H, d_k]; v [T, H, d_v]; beta [T, H];
    cu_seqlens [N+1] (int); S0 [N, H, d_k, d_v] or None (zero state).
    Returns ``(o [T, H, d_v], S_final [N, H, d_k, d_v])`` as float64 arrays.
    Inputs may be any array-likes (numpy, CPU torch); they are widened to fp64.
    """
    lib = lib or load_library()
    q = _f64(q)
    T, H, dk = q.shape
    k = _f64(k, (T, H, dk))
    la = _f64(log_alpha, (T, H, dk))
    v = _f64(v)
    dv = v.shape[2]
    assert v.shape == (T, H, dv)
    b = _f64(beta, (T, H))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[-1] != T:
        raise ValueError("cu_seqlens[-1] must equal the number of tokens")
    s0 = None if S0 is None else _f64(S0, (N, H, dk, dv))
    o = np.zeros((T, H, dv), dtype=np.float64)
    S = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = lib.kda_oracle_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
                                None if s0 is None else s0.ctypes.data,
                                cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                N, H, dk, dv, _ptr(o), _ptr(S), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, S


def decode_step(q, k, v, log_alpha, beta, S, nthreads: int = 0, lib=None):
    """One recurrent step for B independent sequences (one token each).

    Shapes: q, k, log_alpha [B, H, d_k]; v [B, H, d_v]; beta [B, H];
    S [B, H, d_k, d_v].  Returns ``(o [B, H, d_v], S_new)`` in float64.
    It is the recurrence applied to sequences of length one.
    """
    q = _f64(q)
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return prefill(q, k, v, log_alpha, beta, cu, S0=S, nthreads=nthreads, lib=lib)


def _load_bwd():
    global _bwd_lib
    with _lock:
        if _bwd_lib is None:
            build()
            lib = ctypes.CDLL(_BWD_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_oracle_backward.restype = ctypes.c_int
            lib.kda_oracle_backward.argtypes = [dp, dp, dp, dp, dp, ctypes.c_void_p, dp, ctypes.c_void_p,
                                                ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp,
                                                ctypes.c_int]
            _bwd_lib = lib
    return _bwd_lib


def backward(q, k, v, log_alpha, beta, cu_seqlens, dO, S0=None, dS_final=None, nthreads: int = 0):
    """Exact fp64 gradients of sum <dO, o> + <dS_final, S_final> through the recurrence.

    Shapes as in :func:`prefill`, plus dO [T, H, d_v] and dS_final [N, H, d_k, d_v] (None = 0).
    Returns a dict with dq, dk, dv, dlog_alpha, dbeta, dS0 (float64).
    """
    lib = _load_bwd()
    q = _f64(q)
    T, H, dk = q.shape
    k = _f64(k, (T, H, dk))
    la = _f64(log_alpha, (T, H, dk))
    v = _f64(v)
    dv = v.shape[2]
    b = _f64(beta, (T, H))
    do = _f64(dO, (T, H, dv))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[-1] != T:
        raise ValueError("cu_seqlens[-1] must equal the number of tokens")
    s0 = None if S0 is None else _f64(S0, (N, H, dk, dv))
    dsf = None if dS_final is None else _f64(dS_final, (N, H, dk, dv))
    out = dict(dq=np.zeros((T, H, dk)), dk=np.zeros((T, H, dk)), dv=np.zeros((T, H, dv)),
               dlog_alpha=np.zeros((T, H, dk)), dbeta=np.zeros((T, H)), dS0=np.zeros((N, H, dk, dv)))
    rc = lib.kda_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
                                 None if s0 is None else s0.ctypes.data, _ptr(do),
                                 None if dsf is None else dsf.ctypes.data,
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, H, dk, dv,
                                 _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
                                 _ptr(out["dbeta"]), _ptr(out["dS0"]), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out
