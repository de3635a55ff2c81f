"""Benchmark of the B200 KDA operator: prefill tokens/s (headline) and decode us/step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ``kda_prefill`` call over the whole workload (every sequence and
head), inputs resident in HBM.  The default workload is ``batched_prefill``
(8 sequences x 8192 tokens, H = 32, d_k = d_v = 128, bf16 q/k/v, fp32 gates and
state).  The decode workload (256 sequences x 32 heads, 64 consecutive steps) is
timed in the same run and reported under ``decode``.

With N > 1 (one process per GPU under torchrun) every rank runs its own copy of
the workload (the operator's (sequence, head) units are independent, so there is
no collective on the data path): weak scaling, value = all ranks' tokens / max
rank time.

``--impl reference`` times the fp64 CPU oracle (the only reference this operator
has) on the host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gated_delta_rule_126_b200 import inputs  # noqa: E402

METRIC = "KDA prefill tokens/s & decode µs/step (H=32,d=128) on 1 B200; % of roofline"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Algorithmic work per head-token of prefill at chunk C = 64, d = 128, and per
# head-step of decode (derivation in the design notes):
#   flops = 5*C*d + 6*d^2 (causal C x C products at half, three state products);
#   bytes = q,k,v bf16 + log alpha f32 + beta f32 + o bf16.
def prefill_flops_per_head_token(C, d):
    return 5 * C * d + 6 * d * d


def prefill_bytes_per_head_token(dk, dv, qkv_bytes):
    return (2 * dk + dv) * qkv_bytes + 4 * dk + 4 + dv * qkv_bytes


def decode_bytes_per_head_step(dk, dv, qkv_bytes):
    return 2 * 4 * dk * dv + prefill_bytes_per_head_token(dk, dv, qkv_bytes)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu capture per
# kernel, with the SHA-256 of the kernel's source file at capture time.  A launch's
# traffic is the capture's bytes scaled by the units (head-tokens) the launch
# processes, and is reported as null once the source differs from the captured one.
# Prefill: one launch on 2 x 8192 tokens x 32 heads (524,288 head-tokens).
MEASURED_TRAFFIC = {
    "prefill_tc": {"source": "gated_delta_rule_126_b200/csrc/kda_prefill_tc.cu",
                   "sha256": "2cefdd81b3f23a40798ee9431f8c194622fadb610fd0ecc148454e5ec3f58842",
                   "units": 2 * 8192 * 32, "dram_bytes": 673340416 + 120702976},
}


def measured_traffic(kernel, units):
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None:
        return None
    try:
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    if digest != rec["sha256"]:
        return None
    return rec["dram_bytes"] * units / rec["units"]


def prefill_launches(seqlens, H, tc_path, sms=148):
    """Kernel launches of one kda_prefill call: the ordering kernel and the prefill.  On the
    tensor-core path long sequences are split: up to m = min(T / 16384, 8, 2 sms / (3 H))
    sequences of at least 16,384 tokens with 2 L sms > 3 T H (longest first), each cut
    into nseg segments (the most with m H (2 nseg - 3) <= sms, within [3, 8], segments of
    at least 4096 tokens).  That adds nseg - 2 launches of the start-state chain, a second
    prefill pass and the plain sequences' own launch (the chain runs on its side stream)."""
    T = sum(seqlens)
    if not tc_path:
        return 2
    m_max = min(T // 16384, 8, 2 * sms // (3 * max(H, 1)))
    picked = sorted((L for L in seqlens if L >= 16384 and 2 * L * sms > 3 * T * H), reverse=True)[:m_max]
    if not picked:
        return 2
    m = len(picked)
    nseg = max(3, min((sms // (m * H) + 3) // 2, min(picked) // 4096, 8))
    return nseg + 2


def workload_config(w, world):
    """The ``config`` object of the JSON line: the same for both arms."""
    N = len(w.seqlens)
    return {"workload": w.name, "num_seqs": N,
            "seq_lens": "x".join(str(x) for x in sorted(set(w.seqlens))) if N < 10 else f"{N} varlen",
            "total_tokens_per_gpu": w.total_tokens, "H": w.H, "d_k": w.dk, "d_v": w.dv,
            "chunk": w.chunk, "qkv": w.dtype, "state": "fp32", "gates": "fp32",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (no flush)"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons while the timed
    region runs, through read-only NVML queries in a background thread
    (``nvmlDeviceGetClockInfo``, ``nvmlDeviceGetMaxClockInfo``,
    ``nvmlDeviceGetCurrentClocksEventReasons``); ``nvidia-smi --query-gpu`` is the
    fallback when NVML cannot be loaded.  Only samples taken between ``mark_start()``
    and ``mark_end()`` (the timed region) enter the summary.  Nothing here changes a
    setting of the GPU."""

    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clock-event reason bits (nvml.h): SwPowerCap 0x4, HwSlowdown 0x8,
    # SwThermalSlowdown 0x20, HwThermalSlowdown 0x40
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}
    SMI_FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
                  "clocks_event_reasons.hw_thermal_slowdown",
                  "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index, period_s=0.002):
        self.index = index
        self.period = period_s
        self.samples = []  # (perf_counter, sm_mhz, max_mhz, set of reasons)
        self.source = None
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._handle = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        handle = None
        try:  # the CUDA device's PCI bus id names the same GPU in NVML
            props = torch.cuda.get_device_properties(self.index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            handle = None
        if handle is None:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [x for x in vis.split(",") if x.strip()]
            idx = int(ids[self.index]) if self.index < len(ids) and ids[self.index].strip().isdigit() else self.index
            handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
        return pynvml, handle

    def _reasons_nvml(self):
        nv = self._nvml
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        bits = int(fn(self._handle))
        return {n for n, b in self.BITS.items() if bits & b}

    def _poll_nvml(self):
        nv, h = self._nvml, self._handle
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                self.samples.append((time.perf_counter(), sm, mx, self._reasons_nvml()))
            except Exception:
                pass
            time.sleep(self.period)

    def _poll_smi(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index),
                                      f"--query-gpu={','.join(self.SMI_FIELDS)}",
                                      "--format=csv,noheader,nounits"],
                                     capture_output=True, text=True, timeout=5).stdout
                parts = [p.strip() for p in out.strip().split(",")]
                if len(parts) == len(self.SMI_FIELDS):
                    reasons = {n for n, v in zip(self.NAMES, parts[2:]) if v.lower() == "active"}
                    self.samples.append((time.perf_counter(), float(parts[0]), float(parts[1]), reasons))
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        try:
            self._nvml, self._handle = self._nvml_handle()
            self.source = "nvml"
            target = self._poll_nvml
        except Exception:
            self.source = "nvidia-smi"
            target = self._poll_smi
        self._thread = threading.Thread(target=target, daemon=True)
        self._thread.start()
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=10)
        if self.source == "nvml":
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
        return False

    def summary(self):
        lo = self.t0 if self.t0 is not None else float("-inf")
        hi = self.t1 if self.t1 is not None else float("inf")
        win = [x for x in self.samples if lo <= x[0] <= hi]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = set()
        for x in win:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in win), "sm_max_mhz": max(x[2] for x in win),
                "reasons": sorted(reasons), "samples": len(win), "source": self.source}


def dist_setup(backend="nccl"):
    """Join the process group that torchrun describes in the environment (one rank
    per GPU); a single process needs none.  Returns (world, rank, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def time_region(fn, steps, stream, clock=None):
    """Device time of ``steps`` calls of fn, CUDA events on the launching stream.
    ``clock`` (a running ClockSampler) is told where the region starts and ends."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if clock is not None:
        clock.mark_start()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    if clock is not None:
        clock.mark_end()
    return start.elapsed_time(end) / 1e3


def max_over_ranks(x, world, device="cuda"):
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world, cuda=True):
    if world > 1:
        torch.distributed.barrier()
    if cuda:
        torch.cuda.synchronize()


def weak_scaling_value(tokens_per_rank, steps, max_elapsed_s, world):
    """Whole-job tokens/s: every rank runs its own copy of the workload."""
    return world * tokens_per_rank * steps / max_elapsed_s


def oracle_sample(w, budget_head_tokens, seed_device="cpu"):
    """Time the fp64 oracle on a bounded sample of workload w (host cores).

    The sample is whole sequences of the workload's packing, in order, on all H
    heads, until ``budget_head_tokens`` head-tokens are covered; a sequence longer
    than a sixteenth of the budget is skipped, so the sample holds at least 16
    (sequence, head) units to spread over the worker threads.  Inputs are drawn with the same recipe on the CPU.
    Returns (tokens/s, cores, description, seconds); a token counts all H heads.
    """
    import oracle
    H = w.H
    chosen, tok = [], 0
    for L in w.seqlens:
        if L > max(budget_head_tokens // 16, 1):
            continue
        if tok + L * H > budget_head_tokens and chosen:
            break
        chosen.append(L)
        tok += L * H
    if not chosen:  # every sequence is long: take a prefix of the first one
        chosen = [max(1, budget_head_tokens // H)]
    inp = inputs.prefill_inputs(chosen, H, w.dk, w.dv, w.dtype, w.s0_std, w.seed,
                                device=seed_device)
    f64 = lambda t: t.to(torch.float64).numpy()
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["log_alpha"]),
                   f64(inp["beta"]), inp["cu_seqlens_host"],
                   S0=None if inp["S0"] is None else f64(inp["S0"]), nthreads=cores)
    dt = time.perf_counter() - t0
    value = sum(chosen) / dt
    sample = (f"{len(chosen)} sequence(s) ({min(chosen)}..{max(chosen)} tokens) x {H} heads "
              f"= {sum(chosen) * H} head-tokens, fp64 oracle, {dt:.1f} s on {cores} threads")
    return value, cores, sample, dt


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = inputs.WORKLOADS[args.workload]
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, sample, _ = oracle_sample(w, args.ref_head_tokens)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    total_tokens = sum(w.seqlens)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_tokens / value * 1e3,
            "ms_per_step_basis": "the workload's tokens at the sample's rate (each step times a bounded sample)",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world), "sample": sample,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    from gated_delta_rule_126_b200 import (backward_workspace_size, kda_backward, kda_decode_step,
                                           kda_decode_tokens, kda_prefill, kda_prefill_gated, kda_prologue,
                                           prefill_workspace_size)
    world, rank, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks, peak_kind = load_peaks()
    w = inputs.WORKLOADS[args.workload]
    assert w.kind == "prefill"
    inp = inputs.prefill_inputs(w.seqlens, w.H, w.dk, w.dv, w.dtype, w.s0_std,
                                w.seed + 1000 * rank, device=dev)
    T, N = w.total_tokens, len(w.seqlens)
    o = torch.empty(T, w.H, w.dv, dtype=inp["q"].dtype, device=dev)
    S_final = torch.empty(N, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)
    ws = torch.empty(max(256, prefill_workspace_size(N, T, w.H, w.dk, w.dv, w.chunk,
                                                     inp["q"].dtype)),
                     dtype=torch.uint8, device=dev)
    cu_host = inp["cu_seqlens_host"]

    def step():
        kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                    inp["cu_seqlens"], cu_host, S0=inp["S0"], chunk=w.chunk, o=o,
                    S_final=S_final, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    barrier(world)
    with ClockSampler(local) as clk:
        elapsed = time_region(step, args.steps, stream, clock=clk)
    barrier(world)
    elapsed = max_over_ranks(elapsed, world)
    ms = elapsed / args.steps * 1e3
    value = weak_scaling_value(T, args.steps, elapsed, world)

    # roofline of the prefill kernel (one launch per step; events above bracket the
    # call, which also holds a one-thread-block ordering kernel of a few microseconds)
    qkv_bytes = inp["q"].element_size()
    head_tokens = T * w.H
    alg_bytes = head_tokens * prefill_bytes_per_head_token(w.dk, w.dv, qkv_bytes)
    alg_bytes += N * w.H * w.dk * w.dv * 4 * (2 if inp["S0"] is not None else 1)
    alg_flops = head_tokens * prefill_flops_per_head_token(w.chunk, w.dk)
    t_launch = elapsed / args.steps
    hbm_peak = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops"]
    achieved_gbs = alg_bytes / t_launch / 1e9
    achieved_tf = alg_flops / t_launch / 1e12
    t_roof = max(alg_bytes / (hbm_peak * 1e9), alg_flops / (tc_peak * 1e12))
    traffic = measured_traffic("prefill_tc", head_tokens) if w.dtype == "bf16" else None
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                "peak_source": f"{peak_kind} hbm_gbs (copy, burst)",
                "alg_bytes_per_launch": alg_bytes, "alg_flops_per_launch": alg_flops,
                "tensor": {"achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                           "frac": achieved_tf / tc_peak,
                           "peak_source": f"{peak_kind} bf16_tflops (burst)"},
                "frac_of_max_bound": t_roof / t_launch}

    # end to end through the public API: pinned host inputs -> device -> kda_prefill ->
    # host outputs, every step
    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "log_alpha", "beta"]
        host = {n: inp[n].cpu().pin_memory() for n in names}
        h_s0 = inp["S0"].cpu().pin_memory() if inp["S0"] is not None else None
        h_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h_S = torch.empty(S_final.shape, dtype=S_final.dtype, pin_memory=True)
        dbuf = {n: torch.empty_like(inp[n]) for n in names}
        d_s0 = torch.empty_like(inp["S0"]) if inp["S0"] is not None else None
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        h2d += 0 if h_s0 is None else h_s0.numel() * 4
        h2d += len(cu_host) * 4
        d2h = h_o.numel() * h_o.element_size() + h_S.numel() * 4
        cu_pinned = torch.tensor(cu_host, dtype=torch.int32).pin_memory()
        d_cu = torch.empty_like(inp["cu_seqlens"])

        def e2e_step():
            for n in names:
                dbuf[n].copy_(host[n], non_blocking=True)
            if d_s0 is not None:
                d_s0.copy_(h_s0, non_blocking=True)
            d_cu.copy_(cu_pinned, non_blocking=True)
            kda_prefill(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"],
                        d_cu, cu_host, S0=d_s0, chunk=w.chunk, o=o, S_final=S_final,
                        workspace=ws, stream=stream)
            h_o.copy_(o, non_blocking=True)
            h_S.copy_(S_final, non_blocking=True)

        e2e_step()
        barrier(world)
        e_steps = max(1, min(args.steps, 5))
        e_el = max_over_ranks(time_region(e2e_step, e_steps, stream), world)
        e2e = {"value": world * T * e_steps / e_el, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": e_steps}
        del host, dbuf, h_o, h_S

    # the same prefill with the layer's output epilogue (sigmoid gate + RMSNorm) fused
    # into the output store: one more bf16 read (the gate) per head-token, same launches
    gated = None
    if not args.no_gated and w.dtype == "bf16" and w.dk == 128 and w.dv == 128 and w.chunk == 64:
        gate, g_w = inputs.gate_inputs(T, w.H, w.dv, w.dtype, seed=w.seed + 7 + 1000 * rank, device=dev)
        y = torch.empty_like(o)

        def gstep():
            kda_prefill_gated(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              inp["cu_seqlens"], gate, g_w, 1e-6, cu_seqlens_host=cu_host,
                              S0=inp["S0"], chunk=w.chunk, y=y, S_final=S_final, workspace=ws,
                              stream=stream)

        for _ in range(args.warmup):
            gstep()
        barrier(world)
        g_el = max_over_ranks(time_region(gstep, args.steps, stream), world)
        g_t = g_el / args.steps
        g_bytes = alg_bytes + head_tokens * w.dv * qkv_bytes
        g_gbs = g_bytes / g_t / 1e9
        gated = {"value": weak_scaling_value(T, args.steps, g_el, world), "unit": UNIT,
                 "ms_per_step": g_t * 1e3, "epilogue": "y = o / sqrt(mean(o^2) + 1e-6) * w * sigmoid(gate)",
                 "gpu_launches_per_step": 2,
                 "roofline": {"bound": "hbm", "achieved": g_gbs, "peak": hbm_peak, "unit": "GB/s",
                              "frac": g_gbs / hbm_peak, "alg_bytes_per_launch": g_bytes}}
        del gate, g_w, y

    # the layer's input prologue (short conv + Swish + L2Norm, gates) that makes this
    # workload's prefill inputs from its projections: one HBM-bound launch
    prologue = None
    if not args.no_prologue and w.dk % 4 == 0 and w.dv % 4 == 0:
        pin = inputs.prologue_inputs(w.seqlens, w.H, w.dk, w.dv, w.dtype, width=4,
                                     seed=w.seed + 11 + 1000 * rank, device=dev)
        pout = {n: torch.empty_like(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")}

        def pstep():
            kda_prologue(pin["q_pre"], pin["k_pre"], pin["v_pre"], pin["conv_q"], pin["conv_k"],
                         pin["conv_v"], pin["a_gate"], pin["rate"], pin["b_gate"], pin["cu_seqlens"],
                         cu_seqlens_host=cu_host, out=pout, stream=stream)

        for _ in range(args.warmup):
            pstep()
        barrier(world)
        p_el = max_over_ranks(time_region(pstep, args.steps, stream), world)
        p_t = p_el / args.steps
        # bytes per head-token: q/k/v projections in and q/k/v out (dtype), a_gate in and
        # log alpha out (f32), b_gate in and beta out (f32)
        p_bytes = head_tokens * 2 * ((2 * w.dk + w.dv) * qkv_bytes + 4 * w.dk + 4)
        p_gbs = p_bytes / p_t / 1e9
        prologue = {"value": weak_scaling_value(T, args.steps, p_el, world), "unit": UNIT,
                    "ms_per_step": p_t * 1e3, "conv_width": 4, "gpu_launches_per_step": 1,
                    "roofline": {"bound": "hbm", "achieved": p_gbs, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": p_gbs / hbm_peak, "alg_bytes_per_launch": p_bytes}}
        del pin, pout

    # the backward pass (training) on the same batch: dO and dS_final given, gradients of
    # q, k, v, log alpha, beta and S0 out; two kernels (forward sweep with checkpoints,
    # backward sweep adding its value-column slices' sums into the zeroed outputs) after
    # four memsets, float32 on CUDA cores
    backward = None
    if not args.no_backward:
        dO, dSf = inputs.grad_inputs(T, N, w.H, w.dk, w.dv, w.dtype, seed=w.seed + 13 + 1000 * rank,
                                     device=dev)
        bws = torch.empty(max(256, backward_workspace_size(N, T, w.H, w.dk, w.dv)), dtype=torch.uint8,
                          device=dev)

        def bstep():
            kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["cu_seqlens"], dO,
                         cu_seqlens_host=cu_host, S0=inp["S0"], dS_final=dSf, workspace=bws, stream=stream)

        for _ in range(args.warmup):
            bstep()
        barrier(world)
        b_steps = max(1, min(args.steps, 5))
        b_el = max_over_ranks(time_region(bstep, b_steps, stream), world)
        b_t = b_el / b_steps
        # flops per state element and token: forward sweep 5 (decay, P^T k, rank-1 update),
        # adjoint 18 (P, S_t, G += q do^T, S_t do, G e, G^T k, dP, P du, dP.P, alpha dP)
        b_flops = head_tokens * w.dk * w.dv * 23
        b_tf = b_flops / b_t / 1e12
        sm_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        alu_peak = sms * 128 * 2 * sm_mhz * 1e6 / 1e12
        backward = {"value": weak_scaling_value(T, b_steps, b_el, world), "unit": UNIT,
                    "ms_per_step": b_t * 1e3, "steps": b_steps, "gpu_launches_per_step": 2,
                    "grads": "dq, dk, dv, dlog_alpha, dbeta, dS0 (float32)",
                    "roofline": {"bound": "alu", "achieved": b_tf, "peak": alu_peak, "unit": "TFLOP/s",
                                 "frac": b_tf / alu_peak, "alg_flops_per_launch": b_flops,
                                 "peak_source": f"derived: {sms} SMs x 128 fp32 lanes x 2 flops x {sm_mhz:.0f} MHz"}}
        del dO, dSf, bws

    # decode: 256 sequences x 32 heads, 64 consecutive one-token steps
    decode = None
    if not args.no_decode:
        dw = inputs.WORKLOADS["decode"]
        dinp = inputs.workload_inputs(dw, device=dev)
        S = dinp["S0"].clone()
        od = torch.empty(dw.batch, dw.H, dw.dv, dtype=dinp["q"].dtype, device=dev)

        def dstep_all():
            for t in range(dw.steps):
                kda_decode_step(dinp["q"][t], dinp["k"][t], dinp["v"][t], dinp["log_alpha"][t],
                                dinp["beta"][t], S, o=od, stream=stream)

        dstep_all()
        barrier(world)
        d_el = max_over_ranks(time_region(dstep_all, 3, stream), world)
        us = d_el / (3 * dw.steps) * 1e6
        dbytes = dw.batch * dw.H * decode_bytes_per_head_step(dw.dk, dw.dv, 2)
        gbs = dbytes / (us * 1e-6) / 1e9
        # serving form: 4 tokens per call for the same 256 x 32 sequences, states in a
        # slot pool addressed through a permuted slot table (each state crosses HBM
        # once per call instead of once per token)
        n_tok = 4
        tin = inputs.decode_inputs(dw.batch * n_tok, dw.H, dw.dk, dw.dv, 1, dw.dtype,
                                   seed=dw.seed + 7, device=dev)
        tq = {n_: tin[n_][0].reshape(dw.batch, n_tok, dw.H, -1).contiguous()
              for n_ in ("q", "k", "v", "log_alpha")}
        tbeta = tin["beta"][0].reshape(dw.batch, n_tok, dw.H).contiguous()
        pool = tin["S0"][:dw.batch].clone()
        slots = torch.randperm(dw.batch, generator=torch.Generator().manual_seed(3)).to(
            torch.int32).to(dev)
        otok = torch.empty(dw.batch, n_tok, dw.H, dw.dv, dtype=tq["q"].dtype, device=dev)

        def dtok():
            kda_decode_tokens(tq["q"], tq["k"], tq["v"], tq["log_alpha"], tbeta, pool, slots,
                              o=otok, stream=stream)

        for _ in range(3):
            dtok()
        barrier(world)
        t_el = max_over_ranks(time_region(dtok, 20, stream), world)
        us_call = t_el / 20 * 1e6
        tbytes = dw.batch * dw.H * (2 * 4 * dw.dk * dw.dv +
                                    n_tok * prefill_bytes_per_head_token(dw.dk, dw.dv, 2))
        tgbs = tbytes / (us_call * 1e-6) / 1e9
        decode_tokens = {"tokens_per_call": n_tok, "us_per_call": us_call,
                         "us_per_token": us_call / n_tok,
                         "tokens_per_s": world * dw.batch * n_tok / (us_call * 1e-6),
                         "roofline": {"bound": "hbm", "achieved": tgbs, "peak": hbm_peak,
                                      "unit": "GB/s", "frac": tgbs / hbm_peak,
                                      "alg_bytes_per_launch": tbytes}}
        del tin, tq, pool
        decode = {"workload": dw.name, "us_per_step": us, "batch": dw.batch, "H": dw.H,
                  "steps_per_sequence": dw.steps,
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                               "frac": gbs / hbm_peak, "traffic": None,
                               "alg_bytes_per_launch": dbytes,
                               "peak_source": f"{peak_kind} hbm_gbs (copy, burst)"},
                  "gpu_launches_per_step": 1, "multi_token": decode_tokens}
        del dinp, S

    # the 1,048,576-token long-context packing (one 524,288-token sequence + 64 shorter
    # ones, H = 32), timed like the headline workload; the tensor-core path splits the
    # long sequence into segments that run in parallel
    longctx = None
    if not args.no_longctx and args.workload != "longctx_varlen_prefill":
        lw = inputs.WORKLOADS["longctx_varlen_prefill"]
        linp = inputs.prefill_inputs(lw.seqlens, lw.H, lw.dk, lw.dv, lw.dtype, lw.s0_std,
                                     lw.seed + 1000 * rank, device=dev)
        LT, LN = lw.total_tokens, len(lw.seqlens)
        lo = torch.empty(LT, lw.H, lw.dv, dtype=linp["q"].dtype, device=dev)
        lS = torch.empty(LN, lw.H, lw.dk, lw.dv, dtype=torch.float32, device=dev)
        lws = torch.empty(max(256, prefill_workspace_size(LN, LT, lw.H, lw.dk, lw.dv, lw.chunk,
                                                          linp["q"].dtype)), dtype=torch.uint8, device=dev)

        def lstep():
            kda_prefill(linp["q"], linp["k"], linp["v"], linp["log_alpha"], linp["beta"],
                        linp["cu_seqlens"], linp["cu_seqlens_host"], S0=linp["S0"], chunk=lw.chunk,
                        o=lo, S_final=lS, workspace=lws, stream=stream)

        for _ in range(args.warmup):
            lstep()
        barrier(world)
        l_steps = max(1, min(args.steps, 5))
        l_el = max_over_ranks(time_region(lstep, l_steps, stream), world)
        l_t = l_el / l_steps
        l_bytes = LT * lw.H * prefill_bytes_per_head_token(lw.dk, lw.dv, 2) + LN * lw.H * lw.dk * lw.dv * 4
        l_gbs = l_bytes / l_t / 1e9
        longctx = {"workload": lw.name, "total_tokens": LT, "num_seqs": LN, "longest": max(lw.seqlens),
                   "ms_per_step": l_t * 1e3, "steps": l_steps,
                   "value": weak_scaling_value(LT, l_steps, l_el, world), "unit": UNIT,
                   "gpu_launches_per_step": prefill_launches(lw.seqlens, lw.H, True, sms),
                   "roofline": {"bound": "hbm", "achieved": l_gbs, "peak": hbm_peak, "unit": "GB/s",
                                "frac": l_gbs / hbm_peak, "alg_bytes_per_launch": l_bytes}}
        del linp, lo, lS, lws

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_sample(inputs.WORKLOADS[args.workload], args.ref_head_tokens)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": workload_config(w, world),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": prefill_launches(w.seqlens, w.H, w.dtype == "bf16" and w.dk == 128 and w.dv == 128
                                                 and w.chunk == 64, sms) * args.steps,
                "clocks": clk.summary(), "decode": decode,
                "longctx": longctx, "gated_epilogue": gated, "prologue": prologue, "backward": backward}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="batched_prefill",
                    choices=[k for k, v in inputs.WORKLOADS.items() if v.kind == "prefill"])
    ap.add_argument("--ref-head-tokens", type=int, default=1 << 20,
                    help="size of the oracle's timed sample in head-tokens")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-gated", action="store_true")
    ap.add_argument("--no-prologue", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-longctx", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
