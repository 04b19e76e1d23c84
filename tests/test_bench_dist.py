"""The multi-process side of bench.py on CPU: two gloo ranks (world size 2).

The attention path has no exchange step, so N GPUs run independent replicas;
what bench.py does across ranks is take the slowest rank's time and report the
whole job's throughput.  This checks that logic, and that the reference arm
runs on rank 0 only, without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = [12.5, 20.0][rank]
        m = bench.max_over_ranks(ms, world)
        v = bench.whole_job_tflops(2.0e12, world, 10, m)
        out.put((rank, m, v))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 20.0                                  # the slowest rank's time
        assert v == pytest.approx(2.0e12 * 2 * 10 / 0.020 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(1e12, 1, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank0_only(capsys, monkeypatch):
    import bench

    class A:
        config, steps, warmup, gpus = "c1", 2, 1, 2
    bench.run_reference(A, rank=1)
    assert capsys.readouterr().out == ""
    bench.run_reference(A, rank=0)
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_of_the_backward(capsys):
    """--impl reference --pass bwd: the gradient oracle on whole units."""
    import bench

    class A:
        config, steps, warmup, gpus, pass_ = "c1", 1, 0, 1, "bwd"
    bench.run_reference(A, rank=0)
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC_BWD and line["value"] > 0
    assert line["config"]["pass"] == "bwd" and line["cpu_baseline"]["kind"] == "oracle"
