"""Seeded synthetic inputs for the KDA operator.

This module is shared by the tests, the benchmark and the smoke check; it holds
none of the operator's arithmetic (no decay, no state update, no read-out), only
the input recipe, so that the CUDA path and the CPU oracle can be fed the very
same values.

Recipe (the pages give no dataset for the operator; these shapes follow the
workloads they discuss: H=32 heads of d_k=d_v=128, contexts up to 1M tokens):

* q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32 (the KDA layer
  applies L2Norm to q and k before the operator), then cast to the q/k/v dtype;
* v ~ N(0, 1), cast to the q/k/v dtype;
* log alpha = -0.1 * softplus(N(0, 1)) in fp32, one value per (token, head,
  key channel), so alpha lies in (0, 1];
* beta = sigmoid(N(0, 1)) in fp32, one value per (token, head);
* S0 ~ N(0, s0_std^2) in fp32 (s0_std = 0.1 means variance 0.01), or zeros.

All draws come from one ``torch.Generator`` on the target device seeded with
``seed``; the stream of draws is q, k, v, log alpha, beta, S0 in that order, in
token slices of ``slice_tokens`` so that fp32 temporaries stay bounded.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch
import torch.nn.functional as F

S0_STD = 0.1  # "S0 ~ N(0, 0.01)" read as variance 0.01


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named prefill or decode workload."""
    name: str
    kind: str                 # "prefill" or "decode"
    H: int
    dk: int
    dv: int
    dtype: str                # q/k/v (and o) dtype: "f32" or "bf16"
    s0_std: float             # 0.0 = zero initial state
    seed: int
    chunk: int = 64
    seqlens: tuple = ()       # prefill: length of every packed sequence
    batch: int = 0            # decode: number of sequences
    steps: int = 0            # decode: consecutive one-token steps

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens)) if self.kind == "prefill" else self.batch * self.steps


def longctx_seqlens(seed: int, long_len: int = 524288, n_short: int = 64,
                    lo: int = 1024, hi: int = 16384, total: int = 1048576):
    """One long sequence followed by ``n_short`` sequences filling the rest.

    The short lengths are drawn uniformly in [lo, hi], then scaled down in
    proportion (floor) so they sum to ``total - long_len``; the last one takes
    the remainder.  Drawn with numpy's PCG64 from ``seed`` (host side).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    raw = rng.integers(lo, hi + 1, size=n_short).astype(np.int64)
    rest = total - long_len
    scaled = (raw * rest) // raw.sum()
    scaled[-1] += rest - scaled.sum()
    return (long_len,) + tuple(int(x) for x in scaled)


SEED_BASE = 20251026

WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "prefill", H=1, dk=16, dv=16, dtype="f32",
                         s0_std=0.0, seed=SEED_BASE + 0, chunk=16, seqlens=(64,)),
    "single_seq_prefill": Workload("single_seq_prefill", "prefill", H=4, dk=128, dv=128,
                                   dtype="bf16", s0_std=S0_STD, seed=SEED_BASE + 1,
                                   chunk=64, seqlens=(4096,)),
    "batched_prefill": Workload("batched_prefill", "prefill", H=32, dk=128, dv=128,
                                dtype="bf16", s0_std=0.0, seed=SEED_BASE + 2, chunk=64,
                                seqlens=(8192,) * 8),
    # a quarter of the batched workload (above L2, about 0.8 GB of inputs): the
    # small case the profiler captures
    "batched_prefill_2x8192": Workload("batched_prefill_2x8192", "prefill", H=32, dk=128, dv=128,
                                       dtype="bf16", s0_std=0.0, seed=SEED_BASE + 2, chunk=64,
                                       seqlens=(8192,) * 2),
    # the backward pass's profiler case: 4 x 2048 tokens, 32 heads (inputs above L2,
    # about 4 GB of backward workspace)
    "batched_prefill_4x2048": Workload("batched_prefill_4x2048", "prefill", H=32, dk=128, dv=128,
                                       dtype="bf16", s0_std=0.0, seed=SEED_BASE + 2, chunk=64,
                                       seqlens=(2048,) * 4),
    "decode": Workload("decode", "decode", H=32, dk=128, dv=128, dtype="bf16",
                       s0_std=S0_STD, seed=SEED_BASE + 3, batch=256, steps=64),
    "longctx_varlen_prefill": Workload("longctx_varlen_prefill", "prefill", H=32, dk=128,
                                       dv=128, dtype="bf16", s0_std=0.0,
                                       seed=SEED_BASE + 4, chunk=64,
                                       seqlens=longctx_seqlens(SEED_BASE + 4)),
}

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def prefill_inputs(seqlens, H, dk, dv, dtype="bf16", s0_std=0.0, seed=0,
                   device="cpu", slice_tokens=1 << 16):
    """Packed prefill inputs as a dict of tensors on ``device``.

    Keys: q, k [T,H,dk] (dtype); v [T,H,dv] (dtype); log_alpha [T,H,dk] f32;
    beta [T,H] f32; S0 [N,H,dk,dv] f32 or None; cu_seqlens [N+1] int32 (device)
    and cu_seqlens_host (a Python list of ints).
    """
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    N = len(seqlens)
    dt = torch_dtype(dtype)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    q = torch.empty(T, H, dk, dtype=dt, device=device)
    k = torch.empty(T, H, dk, dtype=dt, device=device)
    v = torch.empty(T, H, dv, dtype=dt, device=device)
    la = torch.empty(T, H, dk, dtype=torch.float32, device=device)
    beta = torch.empty(T, H, dtype=torch.float32, device=device)
    for s in range(0, T, slice_tokens):
        e = min(T, s + slice_tokens)
        n = e - s
        f32 = dict(dtype=torch.float32, device=device, generator=gen)
        q[s:e] = _unit_rows(torch.randn(n, H, dk, **f32)).to(dt)
        k[s:e] = _unit_rows(torch.randn(n, H, dk, **f32)).to(dt)
        v[s:e] = torch.randn(n, H, dv, **f32).to(dt)
        la[s:e] = -0.1 * F.softplus(torch.randn(n, H, dk, **f32))
        beta[s:e] = torch.sigmoid(torch.randn(n, H, **f32))
    S0 = None
    if s0_std > 0:
        S0 = s0_std * torch.randn(N, H, dk, dv, dtype=torch.float32, device=device,
                                  generator=gen)
    cu_host = [0]
    for L in seqlens:
        cu_host.append(cu_host[-1] + L)
    cu = torch.tensor(cu_host, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0, cu_seqlens=cu,
                cu_seqlens_host=cu_host)


def decay_log_alpha(T, H, dk, scale=1.0, zero_frac=0.0, seed=0, device="cpu"):
    """log alpha [T,H,dk] fp32 for decays across the whole range alpha in [0, 1].

    log alpha = -scale * softplus(N(0, 1)); ``scale`` is a float or a per-channel
    tensor [dk] (fast- and slow-forgetting channels side by side).  A fraction
    ``zero_frac`` of the entries, drawn at random, is -inf (alpha = 0: the channel is
    erased at that token).  The workloads use scale 0.1 and no zeros; these stronger
    decays test the chunked paths over the rest of the range.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    sc = torch.as_tensor(scale, dtype=torch.float32, device=device)
    la = -sc * F.softplus(torch.randn(T, H, dk, **f32))
    if zero_frac > 0:
        la = torch.where(torch.rand(T, H, dk, **f32) < zero_frac, torch.full_like(la, float("-inf")), la)
    return la.contiguous()


def gate_inputs(T, H, dv, dtype="bf16", seed=0, device="cpu"):
    """Synthetic inputs of the output epilogue: the gate pre-activation [T,H,dv]
    (dtype, ~ N(0, 1)) and the RMSNorm weight [dv] (float32, ~ 1 + 0.1 N(0, 1)).
    Trained projections do not exist here; these stand in for them."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    gate = torch.randn(T, H, dv, **f32).to(torch_dtype(dtype))
    weight = 1.0 + 0.1 * torch.randn(dv, **f32)
    return gate, weight


def grad_inputs(T, N, H, dk, dv, dtype="bf16", seed=0, device="cpu", ds_std=0.1):
    """Synthetic incoming gradients of the backward pass: dO [T,H,dv] (dtype,
    ~ N(0, 1)) and dS_final [N,H,dk,dv] (float32, ~ ds_std N(0, 1); None when
    ds_std == 0).  No loss exists here; these stand in for its gradients."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    dO = torch.randn(T, H, dv, **f32).to(torch_dtype(dtype))
    dS = ds_std * torch.randn(N, H, dk, dv, **f32) if ds_std > 0 else None
    return dO, dS


def prologue_inputs(seqlens, H, dk, dv, dtype="bf16", width=4, seed=0, device="cpu"):
    """Synthetic inputs of the input prologue, packed like ``prefill_inputs``.

    q_pre, k_pre [T,H,dk], v_pre [T,H,dv] ~ N(0, 1) (dtype); conv_q/conv_k [H,dk,W] and
    conv_v [H,dv,W] ~ N(0, 1/W) float32; a_gate [T,H,dk] ~ N(0, 1); rate = 0.1 per head;
    b_gate [T,H] ~ N(0, 1).  With these, log_alpha = -0.1 softplus(N(0, 1)) and
    beta = sigmoid(N(0, 1)), the gate recipe of ``prefill_inputs``.  Trained weights do
    not exist here; these stand in for them.
    """
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    dt = torch_dtype(dtype)
    cu_host = [0]
    for L in seqlens:
        cu_host.append(cu_host[-1] + L)
    return dict(q_pre=torch.randn(T, H, dk, **f32).to(dt), k_pre=torch.randn(T, H, dk, **f32).to(dt),
                v_pre=torch.randn(T, H, dv, **f32).to(dt),
                conv_q=torch.randn(H, dk, width, **f32) / width ** 0.5,
                conv_k=torch.randn(H, dk, width, **f32) / width ** 0.5,
                conv_v=torch.randn(H, dv, width, **f32) / width ** 0.5,
                a_gate=torch.randn(T, H, dk, **f32), rate=torch.full((H,), 0.1, dtype=torch.float32, device=device),
                b_gate=torch.randn(T, H, **f32),
                cu_seqlens=torch.tensor(cu_host, dtype=torch.int32, device=device), cu_seqlens_host=cu_host)


def decode_inputs(batch, H, dk, dv, steps, dtype="bf16", s0_std=S0_STD, seed=0,
                  device="cpu"):
    """Inputs for ``steps`` consecutive one-token decode steps of ``batch`` sequences.

    Keys: q, k [steps,B,H,dk]; v [steps,B,H,dv]; log_alpha [steps,B,H,dk] f32;
    beta [steps,B,H] f32; S0 [B,H,dk,dv] f32 (zeros when s0_std == 0).
    """
    dt = torch_dtype(dtype)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = _unit_rows(torch.randn(steps, batch, H, dk, **f32)).to(dt)
    k = _unit_rows(torch.randn(steps, batch, H, dk, **f32)).to(dt)
    v = torch.randn(steps, batch, H, dv, **f32).to(dt)
    la = -0.1 * F.softplus(torch.randn(steps, batch, H, dk, **f32))
    beta = torch.sigmoid(torch.randn(steps, batch, H, **f32))
    if s0_std > 0:
        S0 = s0_std * torch.randn(batch, H, dk, dv, **f32)
    else:
        S0 = torch.zeros(batch, H, dk, dv, dtype=torch.float32, device=device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0)


def workload_inputs(w: Workload, device="cpu"):
    """Inputs of a named workload (see ``WORKLOADS``)."""
    if w.kind == "prefill":
        return prefill_inputs(w.seqlens, w.H, w.dk, w.dv, w.dtype, w.s0_std, w.seed, device)
    return decode_inputs(w.batch, w.H, w.dk, w.dv, w.steps, w.dtype, w.s0_std, w.seed, device)
