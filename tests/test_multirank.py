"""The multi-rank plumbing of bench.py on CPU ranks (gloo, world size 2).  The
path has no data exchange: a multi-GPU run is N ranks that each encode and
decode their own copy of the set, and the only collective is the maximum of
their timings; the job's throughput counts every rank's bytes over the
slowest rank's time.  The reference arm runs on rank 0 only."""
import argparse
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        per_rank = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        out = bench.max_over_ranks(per_rank, torch.device("cpu"), world)
        q.put((rank, out, bench.job_gbs(world, 1e9, 4, max(out))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timings_reduce_to_the_maximum_on_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
    for p in ps:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in ps] == [0, 0]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, out, gbs in got:
        assert out == [2.0, 5.0, 0.5]
        assert gbs == pytest.approx(2 * 1e9 * 4 / 5.0 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([3, 1.5], None, 1) == [3.0, 1.5]
    assert bench.job_gbs(1, 2e9, 3, 2.0) == pytest.approx(3.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    args = argparse.Namespace(warmup=1, steps=1, gpus=2)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
