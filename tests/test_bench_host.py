"""Host-side bookkeeping of bench.py that needs no GPU: the traffic figure follows the
captured kernel source only, and the launch count follows the sequence split rule."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_126_b200 import inputs  # noqa: E402


def test_traffic_scales_with_units_while_the_source_matches(monkeypatch):
    import hashlib
    rec = dict(bench.MEASURED_TRAFFIC["prefill_tc"])
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        rec["sha256"] = hashlib.sha256(f.read()).hexdigest()  # a capture of the current source
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "prefill_tc", rec)
    per_unit = rec["dram_bytes"] / rec["units"]
    assert bench.measured_traffic("prefill_tc", rec["units"]) == rec["dram_bytes"]
    assert abs(bench.measured_traffic("prefill_tc", 4 * rec["units"]) - 4 * per_unit * rec["units"]) < 1
    assert bench.measured_traffic("no_such_kernel", 1) is None


def test_traffic_is_null_once_the_source_changed(monkeypatch):
    rec = dict(bench.MEASURED_TRAFFIC["prefill_tc"], sha256="0" * 64)
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "prefill_tc", rec)
    assert bench.measured_traffic("prefill_tc", rec["units"]) is None


def test_launch_count_follows_the_split_rule():
    # batched: 8 x 8192 tokens, nothing long enough to split; long context: one 524,288-token sequence
    assert bench.prefill_launches(inputs.WORKLOADS["batched_prefill"].seqlens, 32, True) == 2
    long = inputs.WORKLOADS["longctx_varlen_prefill"].seqlens
    # order + pass A + start-state chain + pass B + the plain sequences' own launch
    assert bench.prefill_launches(long, 32, True) == 5
    assert bench.prefill_launches(long, 32, False) == 2      # the CUDA-core path does not split
    # 2 L 148 > 3 T H with T = L, H = 1; four 4096-token segments: order, pass A, two chain
    # steps, pass B and the plain launch
    assert bench.prefill_launches([16384], 1, True) == 6
    assert bench.prefill_launches([60000, 300], 2, True) == 10  # eight segments (the most)
    assert bench.prefill_launches([16384], 1, True, sms=1) == 2  # 2 L > 3 L fails on one SM
    assert bench.prefill_launches([16383], 1, True) == 2     # below the minimum length


def test_weak_scaling_value_counts_every_rank():
    assert bench.weak_scaling_value(1000, 10, 2.0, 4) == 1000 * 10 * 4 / 2.0


def test_both_arms_report_the_same_config():
    w = inputs.WORKLOADS["batched_prefill"]
    cfg = bench.workload_config(w, 1)
    assert cfg["num_seqs"] == 8 and cfg["seq_lens"] == "8192" and cfg["state"] == "fp32"
    assert cfg == bench.workload_config(w, 1)  # the reference arm calls the same function
    assert bench.workload_config(w, 4)["parallelism"] == "replicas x4"


def test_clock_summary_keeps_only_the_timed_window():
    clk = bench.ClockSampler(0)
    clk.source = "test"
    clk.samples = [(0.0, 300.0, 1965.0, set()),             # idle, before the region
                   (1.0, 1965.0, 1965.0, set()),
                   (1.5, 1950.0, 1965.0, {"sw_power_cap"}),
                   (3.0, 400.0, 1965.0, {"hw_slowdown"})]     # after the region
    clk.t0, clk.t1 = 0.5, 2.0
    s = clk.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1957.5 and s["reasons"] == ["sw_power_cap"]
    clk.t0, clk.t1 = 5.0, 6.0
    assert clk.summary()["samples"] == 0
