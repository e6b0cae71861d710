"""The N > 1 benchmark path on CPU: world-size-2 gloo ranks.

The hot path has no exchange step, so N GPUs run independent replicas; the
only collective is the timing reduction.  These tests run it on gloo."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r+1) ms for the timed steps and 10-r ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = dict(q.get(timeout=10) for _ in range(2))
    assert results[0] == results[1] == [2.0, 10.0]


def test_job_throughput_is_all_units_over_slowest_rank():
    # 2 replicas x 3 steps x 1e12 flop over 2000 ms -> 3 TFLOP/s
    assert bench.job_throughput(2, 1e12, 3, 2000.0) == pytest.approx(3.0)
    assert bench.job_throughput(1, 1e12, 3, 2000.0) == pytest.approx(1.5)


def test_reference_arm_other_ranks_do_no_work(capsys, monkeypatch):
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: pytest.fail("rank 1 ran work"))
    args = bench.argparse.Namespace(gpus=2, steps=1, warmup=3)
    bench.run_reference(args, bench.wl.WORKLOADS["tiny"], rank=1)
    assert capsys.readouterr().out == ""
