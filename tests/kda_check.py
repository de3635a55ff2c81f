"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare them with the relative L2 error.

Tolerances (relative L2 over the compared tensor, computed in fp64):
* float32 q/k/v:                 o and S <= 1e-5
* bfloat16 q/k/v, fp32 state:    o <= 3e-3, S <= 1e-3
When the reference tensor is zero, the max-abs error must be <= 1e-6.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": dict(o=1e-5, S=1e-5), "bf16": dict(o=3e-3, S=1e-3)}


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.linalg.norm(ref))
    if den == 0.0:  # zero reference: fall back to a max-abs bound of 1e-6
        return 0.0 if float(np.abs(x - ref).max(initial=0.0)) <= 1e-6 else float("inf")
    return float(np.linalg.norm(x - ref)) / den


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_units(inp, units, H):
    """Oracle outputs for the (sequence, head) pairs in ``units``.

    Returns {(n, h): (o [L, d_v], S [d_k, d_v])}; inputs are copied to the host one
    (sequence, head) slice at a time.
    """
    cu = inp["cu_seqlens_host"]
    res = {}
    for n, h in units:
        s, e = cu[n], cu[n + 1]
        sl = lambda t: host64(t[s:e, h:h + 1])
        S0 = None if inp["S0"] is None else host64(inp["S0"][n:n + 1, h:h + 1])
        o, S = oracle.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                              host64(inp["beta"][s:e, h:h + 1]), [0, e - s], S0=S0)
        res[(n, h)] = (o[:, 0], S[0, 0])
    return res


def compare_units(inp, o_gpu, S_gpu, units, dtype):
    """Max rel-L2 of o and S over the sampled units; asserts the tolerances."""
    ref = oracle_units(inp, units, inp["q"].shape[1])
    cu = inp["cu_seqlens_host"]
    worst_o = worst_S = 0.0
    for (n, h), (o_ref, S_ref) in ref.items():
        s, e = cu[n], cu[n + 1]
        if e > s:
            worst_o = max(worst_o, rel_l2(host64(o_gpu[s:e, h]), o_ref))
        worst_S = max(worst_S, rel_l2(host64(S_gpu[n, h]), S_ref))
    tol = TOL[dtype]
    assert worst_o <= tol["o"], f"o rel-L2 {worst_o:.3e} > {tol['o']}"
    assert worst_S <= tol["S"], f"S rel-L2 {worst_S:.3e} > {tol['S']}"
    return worst_o, worst_S


def compare_heads(inp, o_gpu, S_gpu, heads, dtype):
    """Rel-L2 over every sequence of the heads in ``heads``, as one tensor each for o
    and S_final, against the oracle; asserts the tolerances.  The oracle runs one head
    at a time (all sequences of that head in one call, threaded over the sequences), so
    the host holds one head's inputs in fp64 at once."""
    cu = inp["cu_seqlens_host"]
    err = {"o": 0.0, "S": 0.0}
    ref2 = {"o": 0.0, "S": 0.0}
    for h in heads:
        sl = lambda t: host64(t[:, h:h + 1])
        S0 = None if inp["S0"] is None else host64(inp["S0"][:, h:h + 1])
        o_ref, S_ref = oracle.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                                      host64(inp["beta"][:, h:h + 1]), cu, S0=S0)
        for key, x, r in (("o", host64(o_gpu[:, h:h + 1]), o_ref), ("S", host64(S_gpu[:, h:h + 1]), S_ref)):
            err[key] += float(np.sum((x - r) ** 2))
            ref2[key] += float(np.sum(r ** 2))
        del o_ref, S_ref
    worst = {key: (err[key] / ref2[key]) ** 0.5 for key in err}
    tol = TOL[dtype]
    assert worst["o"] <= tol["o"], f"o rel-L2 {worst['o']:.3e} > {tol['o']} over heads {heads}"
    assert worst["S"] <= tol["S"], f"S rel-L2 {worst['S']:.3e} > {tol['S']} over heads {heads}"
    return worst["o"], worst["S"]


def compare_full(inp, o_gpu, S_gpu, dtype):
    """Whole-tensor rel-L2 against the oracle over every (sequence, head)."""
    o_ref, S_ref = oracle.prefill(host64(inp["q"]), host64(inp["k"]), host64(inp["v"]),
                                  host64(inp["log_alpha"]), host64(inp["beta"]),
                                  inp["cu_seqlens_host"],
                                  S0=None if inp["S0"] is None else host64(inp["S0"]))
    eo = rel_l2(host64(o_gpu), o_ref)
    eS = rel_l2(host64(S_gpu), S_ref)
    tol = TOL[dtype]
    assert eo <= tol["o"], f"o rel-L2 {eo:.3e} > {tol['o']}"
    assert eS <= tol["S"], f"S rel-L2 {eS:.3e} > {tol['S']}"
    return eo, eS
