"""Replica runs (bench.py --gpus N, one process per GPU under torchrun): the
cross-rank steps run here on CPU with two gloo ranks — the barrier, the maximum
of the timings over ranks (the job's time is the slowest rank's), the minimum of
the warm-up flag, and the reference arm's rank-0-only rule.  The decode path has
no data-path collective (replicas only), so these are the only exchanges.
"""
from __future__ import annotations

import os
import socket


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier_sync(True, cuda=False)
        mx = bench.over_ranks([1.0 + rank, 5.0 - rank, 2.5], "max", "cpu", True)
        mn = bench.over_ranks([1.0 if rank == 0 else 0.0], "min", "cpu", True)
        bench.barrier_sync(True, cuda=False)
        q.put((rank, mx, mn))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_warmup_flag():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(2):
            rank, mx, mn = q.get(timeout=120)
            results[rank] = (mx, mn)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert all(p.exitcode == 0 for p in procs)
    for rank in (0, 1):
        mx, mn = results[rank]
        assert mx == [2.0, 5.0, 2.5]          # element-wise max over the two ranks
        assert mn == [0.0]                    # warm-up ends only when every rank is done


def test_single_process_reductions_are_identity():
    import bench
    assert bench.over_ranks([3.0, 1.5], "max", "cpu", False) == [3.0, 1.5]
    assert bench.over_ranks([0.0], "min", "cpu", False) == [0.0]


def test_reference_arm_prints_on_rank_zero_only(monkeypatch, capsys):
    import json

    import bench
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                     "--warmup", "0", "--cpu-seconds", "1"])
    args = bench.parse()
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(args)
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out)
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
