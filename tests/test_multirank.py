"""The multi-rank plumbing of bench.py on CPU ranks (gloo, world size 2).  The
path has no data exchange: a multi-GPU run partitions the tensor set, whole
tensors, across the ranks, each rank encodes and decodes its share, and the
only collectives are the maximum of the timings and the sum of the byte
counts; the job's throughput is all bytes over the slowest rank's time.
The reference arm runs on rank 0 only."""
import argparse
import datetime
import hashlib
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(target, world, *extra):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=target, args=(r, world, port, q) + extra) for r in range(world)]
    for p in ps:
        p.start()
    got = [q.get(timeout=300) for _ in range(world)]
    for p in ps:
        p.join(timeout=120)
    for p in ps:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in ps] == [0] * world
    return sorted(got, key=lambda g: g[0])


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    return dist


def _timing_worker(rank, world, port, q):
    import torch
    import bench
    dist = _init(rank, world, port)
    try:
        per_rank = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        out = bench.max_over_ranks(per_rank, torch.device("cpu"), world)
        tot = bench.sum_over_ranks([1e9 * (rank + 1)], torch.device("cpu"), world)
        q.put((rank, out, tot, bench.job_gbs(tot[0], 4, max(out))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timings_reduce_to_the_maximum_and_bytes_to_the_sum():
    for rank, out, tot, gbs in _spawn(_timing_worker, 2):
        assert out == [2.0, 5.0, 0.5]
        assert tot == [3e9]
        assert gbs == pytest.approx(3e9 * 4 / 5.0 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([3, 1.5], None, 1) == [3.0, 1.5]
    assert bench.sum_over_ranks([3, 1.5], None, 1) == [3.0, 1.5]
    assert bench.job_gbs(2e9, 3, 2.0) == pytest.approx(3.0)


def test_line_figures_from_the_timed_steps():
    """legs(): the line's means from the K steps' totals, the per-step median
    and best beside them, roofline fractions from the algorithmic bytes."""
    import bench
    enc_steps, dec_steps = [0.010, 0.012, 0.011], [0.007, 0.0072, 0.0071]
    assert bench.step_stats(enc_steps) == [0.011, 0.010]
    r = bench.legs(15e9, 10e9, 3, 0.06, sum(enc_steps), sum(dec_steps), 6540.0,
                   bench.step_stats(enc_steps), bench.step_stats(dec_steps))
    assert r["ms_per_step"] == pytest.approx(20.0)
    assert r["encode"]["ms"] == pytest.approx(11.0) and r["decode"]["ms"] == pytest.approx(7.1)
    assert (r["encode"]["ms_median"], r["encode"]["ms_best"]) == (pytest.approx(11.0), pytest.approx(10.0))
    assert (r["decode"]["ms_median"], r["decode"]["ms_best"]) == (pytest.approx(7.1), pytest.approx(7.0))
    assert r["decode"]["roofline_frac"] == pytest.approx(25e9 / 0.0071 / 1e9 / 6540.0)
    assert r["ratio"] == pytest.approx(10 / 15)
    assert "ms_median" not in bench.legs(1, 1, 1, 1.0, 0.5, 0.5, 1.0)["encode"]


def test_partition_covers_every_tensor_once_and_balances():
    import bench
    for cid in (2, 3, 4):
        specs = workloads.tensor_specs(cid)
        sizes = [s.numel * s.itemsize for s in specs]
        for world in (1, 2, 3, 4, 8):
            shares = bench.partition(sizes, world)
            flat = sorted(i for s in shares for i in s)
            assert flat == list(range(len(specs)))
            loads = [sum(sizes[i] for i in s) for s in shares]
            # greedy largest-first: no rank exceeds the mean by more than the
            # largest tensor
            assert max(loads) <= sum(sizes) / world + max(sizes)
            assert all(s == sorted(s) for s in shares)
    assert bench.partition([5, 3, 3, 2], 2) == [[0, 3], [1, 2]]


def _oracle_share_worker(rank, world, port, q, cid, n_tensors):
    """Each rank encodes its share of the set with the oracle; rank 0 gathers
    the (index, digest) pairs of all ranks."""
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                                    "oracle"))
    import oracle
    import bench
    dist = _init(rank, world, port)
    try:
        specs = workloads.tensor_specs(cid)[:n_tensors]
        shares = bench.partition([s.numel * s.itemsize for s in specs], world)
        mine = []
        for i in shares[rank]:
            c = oracle.encode(workloads.generate_tensor(cid, i))
            mine.append((i, hashlib.sha256(c.tobytes()).hexdigest()))
        everyone = [None] * world
        dist.all_gather_object(everyone, mine)
        q.put((rank, everyone))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ranks_shares_together_give_every_container(orc):
    """World size 2 on the first 16 tensors of workload 2: the union of the
    ranks' containers is the set's, each equal to the oracle's for that
    tensor, and no tensor is coded twice."""
    cid, n = 2, 16
    got = _spawn(_oracle_share_worker, 2, cid, n)
    for rank, everyone in got:
        pairs = [p for share in everyone for p in share]
        assert sorted(i for i, _ in pairs) == list(range(n))
        for i, h in pairs:
            want = orc.encode(workloads.generate_tensor(cid, i))
            assert h == hashlib.sha256(want.tobytes()).hexdigest(), i


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    args = argparse.Namespace(warmup=1, steps=1, gpus=2, workload=4)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(capsys):
    import json
    import bench
    args = argparse.Namespace(warmup=1, steps=2, gpus=1, workload=1)
    bench.run_reference(args, rank=0, world=1)
    line = json.loads(capsys.readouterr().out)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["cores"] == 1
    assert np.isfinite(line["ms_per_step"])
