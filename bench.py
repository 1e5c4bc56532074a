#!/usr/bin/env python3
"""Throughput of the exponent-plane rANS codec on B200.

One step = the whole hot path over one weight set, inputs resident in HBM:
one batched encode (plane split + histogram + 12-bit table, 32-lane rANS
with raw fallback, offset scan, compaction) and one batched decode (rANS +
plane re-merge) of every tensor.  The headline set is workload 4, the
largest that fits one GPU: 225 bf16 tensors shaped like an 8B dense LM
(hidden 4096, 32 layers, GQA; embedding 128256x4096), 7,504,658,432 values,
15.0 GB, values 0.015 * Student-t(4) (see workloads.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload 4] [--extra 1,2,3,5 | none]

Prints one JSON line (rank 0).  `value` is uncompressed GB per second of
round trip: bytes of all tensors / (encode time + decode time).  Timing:
CUDA events on the launching stream over exactly K steps, barrier +
synchronize on both sides, max over ranks.  The inputs (15 GB) exceed the
126 MB L2, so no flush is needed between steps.  The other workloads are
timed the same way, each for --extra-steps steps, and reported under
`workloads`.

Several GPUs (torchrun): the tensors of the set are partitioned, whole
tensors, across the ranks (largest first, each to the least-loaded rank);
each rank encodes and decodes its share, with no collective on the data
path; the job's time is the slowest rank's, so `value` = all bytes / that
time (total work fixed: strong scaling).

`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

HBM_FALLBACK_GBS = 6650.0
METRIC = "decode & encode GB/s (uncompressed bytes) on 1 B200, % HBM roofline; ratio"
WORKLOAD_NAMES = {
    1: "one bf16 1024x1024 tensor, N(0, 0.02)",
    2: ("bf16 tensor set shaped like a 0.6B decoder LM (hidden 1024, 28 layers, "
        "embedding 151936x1024, 57 norms): 254 tensors"),
    3: "fp32 tensor set shaped like GPT-2 small (12 layers, embedding 50257x768): 49 tensors",
    4: ("bf16 tensor set shaped like an 8B dense LM (hidden 4096, 32 layers, GQA, "
        "embedding 128256x4096), 0.015 * Student-t(4): 225 tensors"),
    5: "adversarial bf16 stream of 2^28 values (uniform, constant, special-value, N(0,1e-3) chunks)",
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=4, choices=[1, 2, 3, 4, 5],
                    help="the headline set")
    ap.add_argument("--extra", default="1,2,3,5",
                    help="other workloads timed after the headline ('none' to skip)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="oracle time budget per worker of the all-cores CPU baseline (0: skip)")
    ap.add_argument("--tensors", type=int, default=0,
                    help="profiling only: use the first N tensors of the set (0: all)")
    ap.add_argument("--no-e2e", action="store_true", help="profiling only: skip the e2e leg")
    ap.add_argument("--no-split12", dest="split12", action="store_false",
                    help="skip the Split12 serving-format leg (wc12_encode / wc12_decode on the "
                         "headline tensors and wc12_linear against cuBLAS bf16, timed after the "
                         "step; the 'split12' object)")
    ap.add_argument("--linear-only", action="store_true",
                    help="profiling only: draw the set's first four gate projections and run the "
                         "wc12_linear leg alone (one JSON line with its 'linear' object)")
    ap.add_argument("--no-dtypes", dest="dtypes", action="store_false",
                    help="skip the fp16 / fp8 leg (the headline set's leading tensors cast on the "
                         "device, batched encode and decode timed; the 'dtypes' object)")
    ap.add_argument("--no-checksum", dest="checksum", action="store_false",
                    help="skip the block-checksum leg (wc_crc32_blocks, 1 MiB blocks, over the "
                         "container arena, timed after the step; the 'checksum' object)")
    return ap.parse_args(argv)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def load_oracle():
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle  # test infrastructure: the CPU baseline / reference arm only
    oracle.build()
    return oracle


# ---------------------------------------------------------------------------
# Partitioning of a tensor set across ranks (whole tensors, no exchange).
def partition(sizes, world: int) -> list[list[int]]:
    """Indices of the tensors each rank codes: largest first, each to the
    rank with the fewest bytes so far (ties to the lower rank); each share
    is returned in set order."""
    load = [0] * world
    shares = [[] for _ in range(world)]
    for i in sorted(range(len(sizes)), key=lambda j: (-sizes[j], j)):
        r = min(range(world), key=lambda q: (load[q], q))
        shares[r].append(i)
        load[r] += sizes[i]
    return [sorted(s) for s in shares]


def max_over_ranks(vals, dev, world):
    """Element-wise maximum of per-rank timings (seconds) over all ranks; every
    rank gets the result.  The only collective of a multi-GPU run: the path
    itself has no exchange (each rank encodes and decodes its own tensors)."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(vals, dev, world):
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def job_gbs(total_bytes, steps, seconds):
    """Whole-job throughput: the bytes all ranks processed over the slowest
    rank's time."""
    return total_bytes * steps / seconds / 1e9


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, one process per host core.
def _oracle_worker(args):
    """Encode + decode the given tensors of a workload with the oracle, over
    and over, until `budget` seconds of oracle time are spent; the tensors
    are drawn first (or arrive drawn) and the timing starts when every worker
    is ready."""
    cid, idx_list, budget, barrier = args[:4]
    given = args[4] if len(args) > 4 else None
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle
    import workloads as wl
    data = given if given is not None else [wl.generate_tensor(cid, i) for i in idx_list]
    oracle.decode(oracle.encode(data[0]))  # loads the library
    if barrier is not None:
        barrier.wait()
    done, spent, j = 0, 0.0, 0
    t0 = time.perf_counter()
    while spent < budget:
        b = data[j % len(data)]
        c = oracle.encode(b)
        back = oracle.decode(c)
        assert np.array_equal(back, b)
        done += b.nbytes
        j += 1
        spent = time.perf_counter() - t0
    return done, spent, j


def cpu_oracle_baseline(cid: int, budget: float, workers: int):
    """GB/s of oracle encode + decode on `workers` processes at once (one per
    host core), each coding its own tensors of workload cid (workload 5, one
    2^28-value tensor: its first 64 chunks, 16 of each kind, drawn once here)."""
    import multiprocessing as mp
    specs = workloads.tensor_specs(cid)
    given = None
    if cid in (2, 4):   # the k and v projections: many equal, modest tensors
        pool_idx = [i for i, s in enumerate(specs) if s.name.endswith((".k", ".v"))]
    elif cid == 5:
        pool_idx = [0]
        given = [workloads.generate_tensor(5, 0)[: 64 * workloads.CHUNK].copy()]
    else:
        pool_idx = [i for i, s in enumerate(specs) if s.numel <= (1 << 22)] or [0]
    ctx = mp.get_context("spawn")
    barrier = ctx.Manager().Barrier(workers)
    assign = [[pool_idx[(w + k * workers) % len(pool_idx)] for k in range(2)] for w in range(workers)]
    with ctx.Pool(workers) as pool:
        res = pool.map(_oracle_worker, [(cid, a, budget, barrier, given) for a in assign])
    total = sum(r[0] for r in res)
    wall = max(r[1] for r in res)
    if given is not None:
        what = "its first 64 chunks (16 of each adversarial kind)"
    else:
        names = sorted({specs[i].name.split(".")[-1] for a in assign for i in a})
        what = f"2 of the {'/'.join(names)} tensors of the set"
    return {"value": total / wall / 1e9, "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": (f"workload {cid}: {workers} processes at once (one per host core), each "
                       f"coding {what} over and over for {budget:.1f} s (encode + decode, "
                       f"{sum(r[2] for r in res)} tensor round trips, {total / 1e9:.2f} GB)")}


def cpu_oracle_single(budget: float):
    """The oracle on one core: workload 1 (one 1024x1024 bf16 tensor)."""
    done, spent, j = _oracle_worker((1, [0], budget, None))
    return {"value": done / spent / 1e9, "unit": "GB/s", "cores": 1,
            "sample": f"workload 1 tensor, {j} encode + decode round trips, {spent:.1f} s"}


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks / throttle reasons, sampled every 20 ms from before
    the warm-up to the end of the timed region; the summary uses the samples
    taken inside the timed region (all of them if fewer than 3 fall there)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        import tempfile
        self.proc = None
        log_dir = os.environ.get("WC_CLOCK_LOG_DIR") or tempfile.gettempdir()
        self.path = os.path.join(log_dir, f"clocks_gpu{gpu_index}_{os.getpid()}.csv")
        self.window = None
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", f"-lms={period_ms}"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.01)

    def mark(self, start: float, end: float):
        self.window = (start, end)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + f[0].split(".")[1]) if "." in f[0] else 0.0
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except (ValueError, IndexError):
                continue
        inside = rows
        if self.window is not None:
            a, b = self.window
            sel = [r for r in rows if a - 0.01 <= r[0] <= b + 0.03]
            if len(sel) >= 3:
                inside = sel
        reasons = set()
        for r in inside:
            for nm, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(nm)
        sm = [r[1] for r in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in inside) if inside else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "period_ms": 20,
                "scope": "timed region" if inside is not rows else "warm-up + timed region"}


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "of measured"
    except (OSError, KeyError, ValueError):
        return HBM_FALLBACK_GBS, "of fallback"


DECODE_SOURCES = ["fp32_weight_compression_b200/csrc/k_decode.cu",
                  "fp32_weight_compression_b200/csrc/wc_format.cuh",
                  "fp32_weight_compression_b200/csrc/wc_block.cuh",
                  "fp32_weight_compression_b200/csrc/wc_planes.cuh"]


ENCODE_SOURCES = ["fp32_weight_compression_b200/csrc/k_hist.cu",
                  "fp32_weight_compression_b200/csrc/k_encode.cu",
                  "fp32_weight_compression_b200/csrc/k_compact.cu",
                  "fp32_weight_compression_b200/csrc/wc_hist.cuh",
                  "fp32_weight_compression_b200/csrc/wc_coder.cuh",
                  "fp32_weight_compression_b200/csrc/wc_format.cuh",
                  "fp32_weight_compression_b200/csrc/wc_block.cuh",
                  "fp32_weight_compression_b200/csrc/wc_planes.cuh"]


def kernel_sources_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: int, src_files, values: int,
                     key: str = "traffic_bytes_per_value") -> float | None:
    """DRAM bytes per launch of `kernel` on the given set, from the ncu
    summary in profiles/ (bytes per value there, times this launch's values),
    valid only while the kernel's sources are unchanged."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_workload{workload}.md")
    if not os.path.exists(path):
        return None
    want, per_value = None, None
    for line in open(path):
        if line.startswith("source_sha256:"):
            want = line.split(":", 1)[1].strip()
        if line.startswith(key + ":"):
            per_value = float(line.split(":", 1)[1].strip())
    if per_value is None or want != kernel_sources_sha(src_files):
        return None
    return per_value * values


# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the host cores,
    rank 0 only.  Each step is a bounded sample of the headline set: one of
    its k projections (4096x1024 bf16, 4.2M values), encode + decode."""
    if rank != 0:
        return
    oracle = load_oracle()
    cid = args.workload
    specs = workloads.tensor_specs(cid)
    k_idx = [i for i, s in enumerate(specs) if s.name.endswith(".k")] or [0]
    data = {}
    for s in range(args.warmup + args.steps):
        i = k_idx[s % len(k_idx)]
        if i not in data and len(data) < 4:
            data[i] = workloads.generate_tensor(cid, i)
    keys = list(data)
    for s in range(args.warmup):
        b = data[keys[s % len(keys)]]
        oracle.decode(oracle.encode(b))
    tot_b, tot_t = 0, 0.0
    for s in range(args.steps):
        b = data[keys[s % len(keys)]]
        t0 = time.perf_counter()
        c = oracle.encode(b)
        back = oracle.decode(c)
        tot_t += time.perf_counter() - t0
        tot_b += b.nbytes
        assert np.array_equal(back, b)
    gbs = tot_b / tot_t / 1e9
    shape = "x".join(str(d) for d in specs[keys[0]].shape)
    sample = (f"per step one {shape} tensor of the set ({len(keys)} k projections in "
              f"rotation), encode + decode, single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "u32",
        "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": WORKLOAD_NAMES[cid], "sample": sample},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def _gen_worker(args):
    cid, i = args
    sys.path.insert(0, ROOT)
    import workloads as wl
    return i, wl.generate_tensor(cid, i)


def generate_pinned(pool, cid, idx):
    """The listed tensors of a workload drawn in the process pool, packed into
    one pinned host buffer (256-byte aligned views).  Returns (buffer, offsets,
    nbytes, numels, dtypes)."""
    import torch
    specs = workloads.tensor_specs(cid)
    offs, off = [], 0
    for i in idx:
        offs.append(off)
        off = (off + specs[i].numel * specs[i].itemsize + 255) // 256 * 256
    host = torch.empty(max(off, 256), dtype=torch.uint8, pin_memory=True)
    hv = host.numpy()
    where = {i: o for i, o in zip(idx, offs)}
    if pool is None:
        it = (_gen_worker((cid, i)) for i in idx)
    else:
        it = pool.imap_unordered(_gen_worker, [(cid, i) for i in idx])
    for i, a in it:
        hv[where[i]:where[i] + a.nbytes] = a.view(np.uint8)
        del a
    nbytes = [specs[i].numel * specs[i].itemsize for i in idx]
    numels = [specs[i].numel for i in idx]
    dts = [torch.bfloat16 if specs[i].dtype == "bf16" else torch.float32 for i in idx]
    return host, offs, nbytes, numels, dts


class DeviceSet:
    """A tensor set resident in HBM with its encoder and decoder bound."""

    def __init__(self, host, offs, nbytes, numels, dts, dev):
        import torch
        from fp32_weight_compression_b200 import wc
        self.dev_in = host.to(dev)
        self.dev_out = torch.zeros_like(self.dev_in)
        self.ins = [self.dev_in[o:o + b].view(d) for o, b, d in zip(offs, nbytes, dts)]
        self.outs = [self.dev_out[o:o + b].view(d) for o, b, d in zip(offs, nbytes, dts)]
        self.enc = wc.BatchEncoder(numels, dts, device=dev)
        self.enc.prepare(self.ins)
        conts_cap = [self.enc.out[o:o + c] for o, c in zip(self.enc.out_offsets, self.enc.caps)]
        self.dec = wc.BatchDecoder(device=dev).prepare(conts_cap, self.outs)
        self.bytes = int(sum(nbytes))
        self.n = len(numels)
        self.launches_per_step = 5 * ((self.n + 255) // 256)   # k_prep, k_hist, k_coder, k_compact, k_decode

    def check(self):
        import torch
        torch.cuda.synchronize()
        self.dec.check()
        assert torch.equal(self.dev_out, self.dev_in), "round trip is not bit-exact"

    def container_bytes(self) -> int:
        return int(self.enc.sizes.sum().item())


def time_steps(ds, K, W, stream, dev, barrier, sampler=None):
    """W warm-up steps, then exactly K timed steps (encode + decode each),
    bracketed by barrier + synchronize.  Returns (total, encode, decode)
    seconds on this rank and the per-step encode and decode seconds."""
    import torch
    for _ in range(max(W, 1)):
        ds.enc.run()
        ds.dec.run()
    ds.check()
    ds.dev_out.zero_()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    start.record(stream)
    for k in range(K):
        ev[k][0].record(stream)
        ds.enc.run()
        ev[k][1].record(stream)
        ds.dec.run()
        ev[k][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier()
    if sampler is not None:
        sampler.mark(t_wall0, t_wall1)
    ds.check()
    t_total = start.elapsed_time(end) / 1e3
    enc_steps = [e[0].elapsed_time(e[1]) / 1e3 for e in ev]
    dec_steps = [e[1].elapsed_time(e[2]) / 1e3 for e in ev]
    return t_total, sum(enc_steps), sum(dec_steps), enc_steps, dec_steps


def step_stats(steps):
    """[median, best] of per-step seconds."""
    return [statistics.median(steps), min(steps)]


def legs(total_in, total_cont, K, t_total, t_enc, t_dec, peak, enc_stats=None, dec_stats=None):
    """The line's figures from the K timed steps; enc_stats / dec_stats:
    [median, best] seconds of one step's encode / decode (added as
    ms_median and ms_best)."""
    enc_bytes = total_in + total_cont  # read input, write container
    dec_bytes = total_cont + total_in  # read container, write output
    r = {
        "value": job_gbs(total_in, K, t_total),
        "ms_per_step": t_total / K * 1e3,
        "encode": {"gbs": job_gbs(total_in, K, t_enc), "ms": t_enc / K * 1e3,
                   "hbm_gbs": job_gbs(enc_bytes, K, t_enc),
                   "roofline_frac": job_gbs(enc_bytes, K, t_enc) / peak},
        "decode": {"gbs": job_gbs(total_in, K, t_dec), "ms": t_dec / K * 1e3,
                   "hbm_gbs": job_gbs(dec_bytes, K, t_dec),
                   "roofline_frac": job_gbs(dec_bytes, K, t_dec) / peak},
        "ratio": total_cont / total_in,
        "dec_bytes": dec_bytes,
    }
    for half, st in (("encode", enc_stats), ("decode", dec_stats)):
        if st is not None:
            r[half]["ms_median"] = st[0] * 1e3
            r[half]["ms_best"] = st[1] * 1e3
    return r


def e2e_leg(args, host, offs, nbytes, dts, dev, stream, barrier, world):
    """End-to-end through the public host API (wc.HostCodec: wc_encode_host /
    wc_decode_host): every step encodes the host-resident inputs (pinned) into
    host containers and decodes those back into host outputs.  The library
    streams windows of tensors through the device with copies in both
    directions overlapping the kernels."""
    import torch
    from fp32_weight_compression_b200 import wc
    hts = [host[o:o + b].view(d) for o, b, d in zip(offs, nbytes, dts)]
    host_out = torch.empty_like(host, pin_memory=True)
    hos = [host_out[o:o + b].view(d) for o, b, d in zip(offs, nbytes, dts)]
    big = max(wc.host_encode_footprint(t.numel(), t.dtype) for t in hts)
    slot = (big + 256 + 255) // 256 * 256
    codec = wc.HostCodec(256 * ((4 * len(hts) + 255) // 256) + 3 * slot, device=dev)
    enc_bufs, sizes = codec.encode_buffers(hts)
    conts = codec.encode(hts, enc_bufs, sizes)      # warm-up + check
    codec.decode(conts, hos)
    assert torch.equal(host_out, host), "end-to-end round trip is not bit-exact"
    host_out.zero_()
    E = max(1, args.e2e_steps)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        conts = codec.encode(hts, enc_bufs, sizes)
        codec.decode(conts, hos)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_e2e = e0.elapsed_time(e1) / 1e3
    assert torch.equal(host_out, host), "end-to-end round trip is not bit-exact"
    total_cont = sum(int(c.numel()) for c in conts)
    del codec, enc_bufs, host_out
    return t_e2e, E, total_cont, len(hts)


# ---------------------------------------------------------------------------
def split12_leg(ins, dev, stream, reps: int = 5):
    """wc12_encode_batch / wc12_decode_batch over every bf16 tensor of the
    set (one call each: six encoder launches, one decoder launch, on a
    stream of its own), containers checked bit-exact.  Algorithmic bytes:
    encode reads the input twice (histogram, pack) and writes the container;
    decode reads the container and writes the values.  For comparison, the
    same work as one wc12_encode / wc12_decode call per tensor, captured in a
    CUDA graph and replayed (`ms_per_tensor_graph`)."""
    import torch
    from fp32_weight_compression_b200 import wc
    L = wc.load()
    ins = [t for t in ins if t.dtype == torch.bfloat16]
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    outs, scrs, sizes = [], [], []
    for t in ins:
        n = t.numel()
        outs.append(torch.empty(wc.split12_encode_bound(n), dtype=torch.uint8, device=dev))
        scrs.append(torch.empty(wc.split12_scratch_bytes(n), dtype=torch.uint8, device=dev))
        sizes.append(torch.zeros(1, dtype=torch.int64, device=dev))
    vals = [torch.empty_like(t) for t in ins]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sh = side.cuda_stream
    eitems = (wc.Split12EncodeItem * len(ins))()
    ditems = (wc.Split12DecodeItem * len(ins))()
    for i, (t, o, sc, z, v) in enumerate(zip(ins, outs, scrs, sizes, vals)):
        eitems[i] = wc.Split12EncodeItem(t.data_ptr(), t.numel(), o.data_ptr(), o.numel(), sc.data_ptr(),
                                         sc.numel(), z.data_ptr())
        ditems[i] = wc.Split12DecodeItem(o.data_ptr(), o.numel(), v.data_ptr(), v.numel())

    def enc():
        wc._check(L.wc12_encode_batch(eitems, len(ins), sh), "wc12_encode_batch")

    def dec():
        wc._check(L.wc12_decode_batch(ditems, len(ins), status.data_ptr(), sh), "wc12_decode_batch")

    def enc_each():
        for t, o, sc, z in zip(ins, outs, scrs, sizes):
            wc._check(L.wc12_encode(t.data_ptr(), t.numel(), o.data_ptr(), o.numel(), sc.data_ptr(),
                                    sc.numel(), z.data_ptr(), sh), "wc12_encode")

    def dec_each():
        for o, v in zip(outs, vals):
            wc._check(L.wc12_decode(o.data_ptr(), o.numel(), v.data_ptr(), 2 * v.numel(),
                                    status.data_ptr(), sh), "wc12_decode")

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(side)
        for _ in range(reps):
            fn()
        b.record(side)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps / 1e3

    with torch.cuda.stream(side):
        enc()
        dec()
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0 and all(torch.equal(a, b) for a, b in zip(vals, ins))
    total = int(sum(int(z.item()) for z in sizes))
    B = sum(t.numel() * 2 for t in ins)
    res = {}
    for name, fn, each, alg in (("encode", enc, enc_each, 2 * B + total), ("decode", dec, dec_each, total + B)):
        with torch.cuda.stream(side):
            fn()
            t = timed(fn)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            each()
        with torch.cuda.stream(side):
            g.replay()
            t_each = timed(g.replay)
        del g
        res[name] = {"ms": t * 1e3, "gbs": B / t / 1e9, "hbm_gbs": alg / t / 1e9,
                     "algorithmic_bytes": alg, "ms_per_tensor_graph": t_each * 1e3}
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0 and all(torch.equal(a, b) for a, b in zip(vals, ins))
    res["ratio"] = total / B
    res["launches"] = {"encode": 6, "decode": 1}
    res["timing"] = ("one batched call per pass, 5 passes; ms_per_tensor_graph: one call per tensor, "
                     "captured in a CUDA graph and replayed")
    del outs, scrs, vals
    return res


def linear_leg(ins, specs_mine, dev, reps: int = 20):
    """wc12_linear (Y = X W^T with W held as a Split12 container, expanded
    into the tensor cores' operand layout inside the kernel) against
    torch.matmul on the bf16 weights (cuBLAS), for token counts M = 1 .. 256
    (the tensor-core path at every M).
    W: the first four gate projections of the set (4096 x 14336 bf16, 117 MB
    each, 470 MB together > L2), used in rotation so that every call reads its
    weights from HBM.  Timed with and without the weights' serving plans
    (wc12_plan, built once before the timing; wc12_linear_planned).  Reported
    per M: microseconds per call and the weight bytes each call reads over
    its time."""
    import torch
    from fp32_weight_compression_b200 import wc
    pick = [i for i, s in enumerate(specs_mine) if s.name.endswith(".gate")][:4]
    if not pick:
        return None
    Ws = [ins[i].view(specs_mine[i].shape) for i in pick]
    N, K = Ws[0].shape
    conts = [wc.split12_encode(w.reshape(-1)) for w in Ws]
    plans = [wc.split12_plan(c, N, K) for c in conts]
    L = wc.load()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = {}
    for M in (1, 2, 4, 8, 16, 64, 256):
        x = torch.randn(M, K, device=dev, dtype=torch.float32).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.float32, device=dev)
        s = torch.cuda.current_stream(dev).cuda_stream

        def ours(r):
            c = conts[r % len(conts)]
            wc._check(L.wc12_linear(c.data_ptr(), c.numel(), N, K, x.data_ptr(), M, y.data_ptr(),
                                    status.data_ptr(), s), "wc12_linear")

        def ours_planned(r):
            c, pl = conts[r % len(conts)], plans[r % len(plans)]
            wc._check(L.wc12_linear_planned(c.data_ptr(), c.numel(), pl.data_ptr(), pl.numel(), N, K,
                                            x.data_ptr(), M, y.data_ptr(), status.data_ptr(), s),
                      "wc12_linear_planned")

        def ref(r):
            torch.matmul(x, Ws[r % len(Ws)].t())

        res = {}
        for name, fn in (("wc12_linear", ours), ("wc12_linear_planned", ours_planned), ("cublas_bf16", ref)):
            for r in range(4):
                fn(r)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a.record()
            for r in range(reps):
                fn(r)
            b.record()
            torch.cuda.synchronize(dev)
            t = a.elapsed_time(b) / reps / 1e3
            wbytes = conts[0].numel() if name.startswith("wc12") else 2 * N * K
            res[name] = {"us": t * 1e6, "weight_gbs": wbytes / t / 1e9}
        assert int(status.item()) == 0
        ref_y = torch.matmul(x.float(), Ws[(reps - 1) % len(Ws)].float().t())
        ours(reps - 1)
        torch.cuda.synchronize(dev)
        res["max_rel_err"] = float(((y - ref_y).abs().max() / ref_y.abs().max().clamp_min(1e-30)).item())
        res["speedup"] = res["cublas_bf16"]["us"] / res["wc12_linear"]["us"]
        res["speedup_planned"] = res["cublas_bf16"]["us"] / res["wc12_linear_planned"]["us"]
        out[str(M)] = res
    return {"N": N, "K": K, "weights": len(Ws), "per_M": out,
            "container_bytes": conts[0].numel(), "plan_bytes": plans[0].numel(), "bf16_bytes": 2 * N * K}


def checksum_leg(arena, dev, stream, reps: int = 10):
    """wc_crc32_blocks over the whole container arena (larger than L2), 1 MiB
    blocks: algorithmic bytes = the arena's bytes read (the CRCs written are
    1/262144 of that)."""
    import torch
    from fp32_weight_compression_b200 import wc
    for _ in range(3):
        wc.crc32_blocks(arena, wc.CRC_BLOCK, stream)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
    torch.cuda.synchronize(dev)
    for r in range(reps):
        evs[2 * r].record(stream)
        wc.crc32_blocks(arena, wc.CRC_BLOCK, stream)
        evs[2 * r + 1].record(stream)
    torch.cuda.synchronize(dev)
    t = sum(evs[2 * r].elapsed_time(evs[2 * r + 1]) for r in range(reps)) / reps / 1e3
    nbytes = arena.numel()
    return {"kernel": "k_crc32", "bytes": nbytes, "block_bytes": wc.CRC_BLOCK, "ms": t * 1e3,
            "gbs": nbytes / t / 1e9, "reps": reps}


def dtypes_leg(ins, dev, stream, budget: int = 600_000_000, reps: int = 5):
    """The other dtypes of the codec (fp16, fp8 e4m3, fp8 e5m2) on the
    headline set's leading bf16 tensors (up to `budget` values), cast on the
    device: one batched encode and one batched decode per dtype, round trip
    checked bit-exact.  Algorithmic bytes: encode reads the input and writes
    the containers, decode reads the containers and writes the values."""
    import torch
    from fp32_weight_compression_b200 import wc
    src, total = [], 0
    for t in ins:
        if t.dtype != torch.bfloat16 or total + t.numel() > budget:
            continue
        src.append(t)
        total += t.numel()
    out = {"values": total, "tensors": len(src)}

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps / 1e3

    for name, dt in (("fp16", torch.float16), ("fp8_e4m3", torch.float8_e4m3fn), ("fp8_e5m2", torch.float8_e5m2)):
        xs = [t.to(dt) for t in src]
        enc = wc.BatchEncoder([x.numel() for x in xs], [x.dtype for x in xs], dev).prepare(xs)
        enc.run(stream)
        torch.cuda.synchronize(dev)
        sizes = enc.sizes.cpu().tolist()
        conts = enc.containers(sizes)
        outs = [torch.empty_like(x) for x in xs]
        dec = wc.BatchDecoder(dev).prepare(conts, outs)
        dec.run(stream)
        torch.cuda.synchronize(dev)
        assert int(dec.status.item()) == 0
        elem = xs[0].element_size()
        ok = all(torch.equal(o.view(torch.uint8), x.view(torch.uint8)) for o, x in zip(outs, xs))
        assert ok, f"{name} round trip"
        B = total * elem
        C = int(sum(sizes))
        te, td = timed(lambda: enc.run(stream)), timed(lambda: dec.run(stream))
        out[name] = {"ratio": C / B,
                     "encode": {"ms": te * 1e3, "gbs": B / te / 1e9, "hbm_gbs": (B + C) / te / 1e9},
                     "decode": {"ms": td * 1e3, "gbs": B / td / 1e9, "hbm_gbs": (B + C) / td / 1e9}}
        del xs, enc, dec, conts, outs
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
def linear_only(cid: int, local: int):
    """The wc12_linear leg on its own (profiling): the set's first four gate
    projections drawn, moved to the device, timed against cuBLAS."""
    import torch
    specs = workloads.tensor_specs(cid)
    pick = [i for i, s in enumerate(specs) if s.name.endswith(".gate")][:4]
    host, offs, nbytes, numels, dts = generate_pinned(None, cid, pick)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ins = [host[o:o + b].to(dev).view(dt) for o, b, dt in zip(offs, nbytes, dts)]
    torch.cuda.synchronize(dev)
    res = linear_leg(ins, [specs[i] for i in pick], dev)
    print(json.dumps({"workload": WORKLOAD_NAMES[cid], "linear": res}))


def main(argv=None):
    args = parse(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    cid = args.workload
    if args.linear_only:
        linear_only(cid, local)
        return
    extra = [] if args.extra in ("", "none") else [int(x) for x in args.extra.split(",")]
    extra = [c for c in extra if c != cid]

    # Host-side work first: the CPU baseline (all cores, then one), the
    # input draw.  Both use spawn-started processes, before any CUDA call.
    cpu_base = None
    cpu_extra = {}  # the other sets' all-core figures, shorter samples
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu_base = cpu_oracle_baseline(cid, args.cpu_seconds, host_cores())
        cpu_base["single_thread"] = cpu_oracle_single(min(3.0, args.cpu_seconds))
        for c in extra:
            cpu_extra[c] = cpu_oracle_baseline(c, min(2.5, args.cpu_seconds), host_cores())
    specs = workloads.tensor_specs(cid)
    idx = list(range(len(specs) if args.tensors <= 0 else min(args.tensors, len(specs))))
    shares = partition([specs[i].numel * specs[i].itemsize for i in idx], world)
    mine = [idx[j] for j in shares[rank]]
    import multiprocessing as mp
    pool = mp.get_context("spawn").Pool(max(1, min(16, host_cores() // max(1, world))))

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    host, offs, nbytes, numels, dts = generate_pinned(pool, cid, mine)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    stream = torch.cuda.current_stream(dev)
    peak, peak_note = peak_hbm()
    ds = DeviceSet(host, offs, nbytes, numels, dts, dev)
    sampler = ClockSampler(local)
    t_total, t_enc, t_dec, enc_steps, dec_steps = time_steps(ds, args.steps, args.warmup, stream, dev,
                                                             barrier, sampler)
    clocks = sampler.stop()
    total_cont = ds.container_bytes()
    t_total, t_enc, t_dec, *st = max_over_ranks(
        [t_total, t_enc, t_dec] + step_stats(enc_steps) + step_stats(dec_steps), dev, world)
    total_in, total_cont = (int(v) for v in sum_over_ranks([ds.bytes, total_cont], dev, world))
    K = args.steps
    r = legs(total_in, total_cont, K, t_total, t_enc, t_dec, peak, st[:2], st[2:])
    values_mine = int(sum(numels))
    checksum = checksum_leg(ds.enc.out, dev, stream) if args.checksum else None
    dtl = dtypes_leg(ds.ins, dev, stream) if args.dtypes and world == 1 else None
    s12 = split12_leg(ds.ins, dev, stream) if args.split12 else None
    if s12 is not None:
        try:
            s12["linear"] = linear_leg(ds.ins, [specs[i] for i in mine], dev)
        except Exception as ex:  # reported, not fatal: the leg is outside the timed step
            s12["linear"] = {"error": f"{type(ex).__name__}: {ex}"[:300]}
    launches = ds.launches_per_step * K
    del ds
    torch.cuda.empty_cache()

    e2e = None
    if not args.no_e2e:
        t_e2e, E, e2e_cont, ntens = e2e_leg(args, host, offs, nbytes, dts, dev, stream, barrier, world)
        t_e2e, = max_over_ranks([t_e2e], dev, world)
        e2e_cont, = sum_over_ranks([e2e_cont], dev, world)
        e2e = {"value": job_gbs(total_in, E, t_e2e), "unit": "GB/s",
               "h2d_bytes_per_step": int(total_in + e2e_cont),
               "d2h_bytes_per_step": int(e2e_cont + 8 * len(idx) + total_in), "steps": E,
               "api": "wc_encode_host + wc_decode_host (pinned host buffers, windows through HBM)"}
    del host

    per_workload = {}
    if world == 1:
        for c in extra:
            cs = workloads.tensor_specs(c)
            h, o, nb, nu, dt = generate_pinned(pool, c, list(range(len(cs))))
            d = DeviceSet(h, o, nb, nu, dt, dev)
            tt, te, td, es, ds_ = time_steps(d, args.extra_steps, 3, stream, dev, barrier)
            rr = legs(d.bytes, d.container_bytes(), args.extra_steps, tt, te, td, peak,
                      step_stats(es), step_stats(ds_))
            rr.pop("dec_bytes")
            rr["workload"] = WORKLOAD_NAMES[c]
            rr["input_bytes"] = d.bytes
            if c in cpu_extra:
                rr["cpu_baseline"] = cpu_extra[c]
            rr["steps"] = args.extra_steps
            per_workload[str(c)] = rr
            launches += d.launches_per_step * args.extra_steps
            del d, h
            torch.cuda.empty_cache()
    pool.close()

    traffic = recorded_traffic("k_decode", cid, DECODE_SOURCES, values_mine) if world == 1 else None
    enc_traffic = (recorded_traffic("k_coder", cid, ENCODE_SOURCES, values_mine, "encode_traffic_bytes_per_value")
                   if world == 1 else None)
    # DRAM bytes of the four encode launches per step, from the recorded ncu
    # capture (null once a kernel source changed): against the algorithmic bytes
    r["encode"]["traffic"] = enc_traffic
    r["encode"]["traffic_over_algorithmic"] = (enc_traffic / (total_in + total_cont)
                                               if enc_traffic else None)
    dec_achieved = r["decode"]["hbm_gbs"]
    line = {
        "metric": METRIC,
        "value": r["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": r["ms_per_step"],
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "u32",
        "data": "synthetic (seeded numpy PCG64; no checkpoints available)",
        "config": {"workload": WORKLOAD_NAMES[cid] + (f" (first {len(idx)})" if args.tensors else ""),
                   "tensors": len(idx), "values": int(sum(specs[i].numel for i in idx)),
                   "input_bytes": total_in,
                   "parallelism": ("one GPU" if world == 1 else
                                   f"tensors partitioned over {world} GPUs (whole tensors, "
                                   f"largest first to the least-loaded rank), no collective"),
                   "l2": f"inputs {total_in / 1e9:.2f} GB > 126 MB L2, no flush"},
        "encode": r["encode"],
        "decode": r["decode"],
        "ratio": r["ratio"],
        "roofline": {"bound": "hbm", "kernel": "k_decode", "achieved": dec_achieved, "peak": peak,
                     "unit": "GB/s", "frac": dec_achieved / peak, "traffic": traffic,
                     "peak_note": peak_note,
                     "algorithmic_bytes_per_launch": r["dec_bytes"] // max(1, world)},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu_base,
        "workloads": per_workload,
    }
    if checksum is not None:
        checksum["roofline_frac"] = checksum["gbs"] / peak
        line["checksum"] = checksum
    if s12 is not None:
        for leg in ("encode", "decode"):
            s12[leg]["roofline_frac"] = s12[leg]["hbm_gbs"] / peak
        line["split12"] = s12
    if dtl is not None:
        for name in ("fp16", "fp8_e4m3", "fp8_e5m2"):
            for leg in ("encode", "decode"):
                dtl[name][leg]["roofline_frac"] = dtl[name][leg]["hbm_gbs"] / peak
        line["dtypes"] = dtl
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
