"""Multi-process path of the benchmark on CPU (gloo, world size 2): each rank
runs an independent replica, the job time is the max over ranks, the value is
all ranks' FLOP over that time, and only rank 0 reports."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        job = bench.job_time_ms(local_ms[rank], world, "cpu")
        value = bench.job_throughput_tflops(1e12, 10, world, job)
        out.put((rank, job, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_ranks_and_value_counts_all_replicas():
    world, port = 2, _free_port()
    local = [12.5, 20.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, job, value in res:
        assert job == 20.0
        assert value == pytest.approx(2 * 10 * 1e12 / 0.020 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.job_time_ms(7.0, 1) == 7.0
    assert bench.job_throughput_tflops(2e12, 5, 1, 10.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_quietly(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"workload": "tiny", "steps": 1, "warmup": 3})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_rank0_prints_the_contract_line(monkeypatch, capsys):
    import json

    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("FA_REFERENCE_STEP_SECONDS", "0.2")
    args = type("A", (), {"workload": "tiny", "steps": 2, "warmup": 3})()
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    assert line["config"]["workload"] == "tiny"
