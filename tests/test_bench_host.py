"""Host-side bookkeeping of bench.py that needs no GPU: the traffic figure follows the
captured kernel source only, and the launch count follows the sequence split rule."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_126_b200 import inputs  # noqa: E402


def test_traffic_scales_with_units_while_the_source_matches():
    rec = bench.MEASURED_TRAFFIC["prefill_tc"]
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
    assert bench.prefill_launches(long, 32, True) == 4
    assert bench.prefill_launches(long, 32, False) == 2      # the CUDA-core path does not split
    assert bench.prefill_launches([16384], 1, True) == 4     # 2 L 148 > 3 T H with T = L, H = 1
    assert bench.prefill_launches([16383], 1, True) == 2     # below the minimum length


def test_weak_scaling_value_counts_every_rank():
    assert bench.weak_scaling_value(1000, 10, 2.0, 4) == 1000 * 10 * 4 / 2.0
