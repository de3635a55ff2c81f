"""The multi-GPU plumbing of bench.py, run as two gloo ranks on the CPU.

bench.py --gpus N runs one process per GPU; every rank processes its own copy of
the workload (the operator's (sequence, head) units never interact), and the job
time is the slowest rank's.  These tests exercise that host logic with the gloo
backend: process-group setup from the torchrun environment, barrier,
max-over-ranks, the weak-scaling value, and the reference arm leaving ranks > 0
without work.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_setup("gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w, cuda=False)
    # each rank "measured" a different time; the job reports the slowest
    elapsed = bench.max_over_ranks(0.5 + rank, w, device="cpu")
    value = bench.weak_scaling_value(65536, 10, elapsed, w)
    out.put((rank, elapsed, value))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_scale_weakly():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, elapsed, value in results:
        assert elapsed == pytest.approx(1.5)          # slowest rank
        assert value == pytest.approx(2 * 65536 * 10 / 1.5)


def test_reference_arm_ranks_above_zero_exit_without_work(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        workload = "batched_prefill"
        steps = 1
        warmup = 3
        ref_head_tokens = 1 << 20

    assert bench.run_reference(Args()) == 0


def test_single_process_needs_no_group(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_setup("gloo") == (1, 0, 0)
    assert bench.max_over_ranks(3.0, 1) == 3.0
