"""Host-side logic of bench.py, on CPU: the max-over-ranks timing reduction
with two gloo ranks (the N > 1 path), the JSON line (weak-scaling
aggregate, roofline fraction, launch count), the step's algorithmic bytes,
and the reference arm's behaviour on ranks other than 0."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out[rank] = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        # every rank takes the same collective steps, then the slowest wins again
        out[world + rank] = bench.max_over_ranks(10.0 - rank, world, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert [out[r] for r in range(world)] == [2.5, 2.5]
        assert [out[world + r] for r in range(world)] == [10.0, 10.0]


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1, None) == 3.25


def test_result_line_weak_scaling_and_roofline():
    step_bytes, n_calls, ms = 7_592_738_816, 448, 5.0
    one = bench.result_line(1, 200, 5, ms, step_bytes, n_calls, {}, 6457.4, "measured", {}, None, None)
    two = bench.result_line(2, 200, 5, ms, step_bytes, n_calls, {}, 6457.4, "measured", {}, None, None)
    assert two["value"] == pytest.approx(2 * one["value"])          # whole-job aggregate
    assert one["value"] == pytest.approx(step_bytes / (ms * 1e6))
    assert one["roofline"]["achieved"] == pytest.approx(one["value"])
    assert two["roofline"]["achieved"] == pytest.approx(one["value"])  # per GPU, not aggregate
    assert one["roofline"]["frac"] == pytest.approx(one["value"] / 6457.4)
    assert one["gpu_launches"] == n_calls * 200
    assert one["scaling"] == "weak" and one["higher_is_better"] is True
    assert one["us_per_call"] == pytest.approx(ms * 1e3 / n_calls)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "vs_baseline",
                "dtype", "data", "config", "roofline", "gpu_launches", "clocks", "e2e", "cpu_baseline"):
        assert key in one
    # the dominant kernel timed on its own sets the roofline, not the step
    dom = {"bytes": 6_000_000_000, "ms": 3.0, "launches": 320}
    three = bench.result_line(1, 200, 5, ms, step_bytes, n_calls, {}, 6457.4, "measured", {}, None, None, dom)
    assert three["value"] == pytest.approx(one["value"])
    assert three["roofline"]["achieved"] == pytest.approx(6_000_000_000 / 3.0e6)
    assert three["roofline"]["launches_per_step"] == 320
    if three["roofline"]["traffic"] is not None:
        assert three["roofline"]["traffic"] == pytest.approx(bench.DRAM_PER_ALGO_BYTE * 6_000_000_000 / 320)


def test_step_bytes_match_the_workload_table():
    calls = bench.stack_calls()
    assert len(calls) == 448
    by_m = {m: sum(bench.algorithmic_bytes(mm, sh.n, sh.k, bench.GROUP) for mm, _, sh in calls if mm == m)
            for m in bench.MS}
    assert by_m[1] == 3_757_047_808 and by_m[16] == 3_835_691_008


def test_reference_arm_other_ranks_do_no_work(capsys):
    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A(), rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_both_arms_share_the_config():
    one = bench.result_line(1, 200, 5, 5.0, 7_592_738_816, 448, {}, 6457.4, "measured", {}, None, None)
    assert one["config"] == bench.bench_config(1)
    assert one["config"]["calls_per_step"] == 448
