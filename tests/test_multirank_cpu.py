"""The N > 1 plumbing of bench.py on CPU: two gloo ranks (replicas only, no
data-path collective).  Every rank must see the slowest rank's time, the
whole-job rate must count every rank's work, and the reference arm's other
ranks must exit without work."""
import argparse
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 * (rank + 1)                 # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, "cpu")
        rate = bench.whole_job_rate(2.0, world, 5, total)
        out.put((rank, total, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]
    # 2 units x 2 ranks x 5 steps in 20 ms
    assert res[0][2] == pytest.approx(2.0 * 2 * 5 / 0.020)


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="llama8b", M=2048, fmt="nvfp4", nm="2:4", residual="own",
                              steps=1, warmup=0, gpus=2)
    called = []
    monkeypatch.setattr(bench, "make_inputs", lambda *a: called.append(a))
    assert bench.run_reference(args) == 0
    assert not called
