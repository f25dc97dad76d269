"""The multi-process bench logic on the CPU: two gloo ranks (one process per
GPU in a real run; here plain processes), replicas only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r "measured" 0.5 + r seconds for 10 steps of 1 token
        el = bench.slowest_rank_time(0.5 + rank, world, "cpu")
        q.put((rank, el, bench.job_throughput(world, 10, 1, el)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_the_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, el, val in got:
        assert el == 1.5                       # the max over ranks, on every rank
        assert val == pytest.approx(2 * 10 / 1.5)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"batch": 1, "warmup": 1, "steps": 1, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""        # no work and no line on other ranks


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.slowest_rank_time(0.25, 1, "cpu") == 0.25
    assert bench.job_throughput(1, 100, 1, 0.25) == 400.0


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    # rank 0 runs the oracle on a bounded sample and prints one JSON line with
    # the arm's keys; its e2e moves no bytes between host and device
    import json

    import bench
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), {"batch": 1, "warmup": 1, "steps": 1, "gpus": 1})()
    assert bench.run_reference(args) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["metric"] == "MoE seed-FFN decode tokens/s" and d["unit"] == "tokens/s"
    assert d["steps"] == 1 and d["n_gpus"] == 1
    assert d["config"] == bench.workload_config(1, 1)   # the GPU arm's config, key for key
    # ms_per_step is the measured time of what a step ran (one layer), which
    # the value scales to the 45-layer stack
    assert d["value"] == pytest.approx(1e3 / (45 * d["ms_per_step"]), rel=1e-3)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert cb["nproc"] >= 1 and cb["cpu_model"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
