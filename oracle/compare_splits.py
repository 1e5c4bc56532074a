"""How much the reorder of the planes is worth: container sizes written by
the oracle for the same seeded weights under different plane splits.

TEST INFRASTRUCTURE ONLY (it runs the CPU oracle; the CUDA library is not
involved).  For each workload's bf16 tensors:
  reorder    dtype 1: exponent byte coded, sign + mantissa byte raw
             ("PTWM", How it works 1-2)
  high byte  dtype 6: bf16 cut into bytes as they are, high byte (sign and
             exponent bits 7..1) coded, low byte raw (the Split12 split of the
             "weight-compression" README)
  split12    the Split12 codec itself (oracle/split12.py): a 4-bit index into
             a 16-entry codebook of high bytes, the low byte raw, exceptions
and, with the values scaled by 64 and rounded to fp8 (torch's CPU casts):
  e4m3       dtype 4: exponent nibble coded
  e5m2       dtype 5: top four exponent bits coded
Prints container bytes / input bytes per split and the coded plane's
empirical entropy (bits per value).

    python oracle/compare_splits.py --workloads 1 2 4 --layers 1
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
import split12  # noqa: E402
import workloads  # noqa: E402


def entropy_bits(plane: np.ndarray) -> float:
    c = np.bincount(plane, minlength=256).astype(np.float64)
    p = c[c > 0] / plane.size
    return float(-(p * np.log2(p)).sum())


def to_fp8(bits16: np.ndarray, kind: str) -> np.ndarray:
    import torch
    x = (bits16.astype(np.uint32) << 16).view(np.float32) * np.float32(64.0)
    dt = torch.float8_e4m3fn if kind == "e4m3" else torch.float8_e5m2
    return torch.from_numpy(x).to(dt).view(torch.uint8).numpy()


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", type=int, nargs="+", default=[1, 2, 4])
    ap.add_argument("--layers", type=int, default=1,
                    help="workload 4: how many of its 32 layers (plus no embedding)")
    args = ap.parse_args()
    oracle.build()
    for cid in args.workloads:
        specs = workloads.tensor_specs(cid)
        idx = list(range(len(specs)))
        if cid == 4:
            idx = idx[: 7 * args.layers]
        tot = {k: 0 for k in ("in", "reorder", "highbyte", "split12", "in8", "e4m3", "e5m2")}
        n_exc = 0
        ent = {k: 0.0 for k in ("reorder", "highbyte", "e4m3", "e5m2")}
        nvals = 0
        for i in idx:
            if specs[i].dtype != "bf16":
                continue
            b = workloads.generate_tensor(cid, i)
            n = b.size
            nvals += n
            tot["in"] += b.nbytes
            tot["reorder"] += oracle.encode(b).size
            tot["highbyte"] += oracle.encode(b, dtype=oracle.BF16_HIGHBYTE).size
            c12 = split12.encode(b)
            tot["split12"] += c12.size
            n_exc += split12.read_header(c12)["ne"]
            ent["reorder"] += entropy_bits(oracle.split_bf16(b)[0]) * n
            ent["highbyte"] += entropy_bits(oracle.split_bf16_highbyte(b)[0]) * n
            for kind, code, split in (("e4m3", oracle.FP8E4M3, oracle.split_fp8e4m3),
                                      ("e5m2", oracle.FP8E5M2, oracle.split_fp8e5m2)):
                f8 = to_fp8(b, kind)
                tot["e4m3" if kind == "e4m3" else "e5m2"] += oracle.encode(f8, dtype=code).size
                ent[kind] += entropy_bits(split(f8)[0]) * n
            tot["in8"] += n
        if not nvals:
            continue
        print(f"workload {cid}: {len(idx)} tensors, {nvals} values")
        print(f"  bf16 reorder    ratio {tot['reorder'] / tot['in']:.4f}  coded plane "
              f"{ent['reorder'] / nvals:.3f} bits/value")
        print(f"  bf16 high byte  ratio {tot['highbyte'] / tot['in']:.4f}  coded plane "
              f"{ent['highbyte'] / nvals:.3f} bits/value")
        print(f"  Split12 codec   ratio {tot['split12'] / tot['in']:.4f}  exceptions "
              f"{100 * n_exc / nvals:.4f} % of values")
        print(f"  fp8 e4m3 (x64)  ratio {tot['e4m3'] / tot['in8']:.4f}  coded plane "
              f"{ent['e4m3'] / nvals:.3f} bits/value")
        print(f"  fp8 e5m2 (x64)  ratio {tot['e5m2'] / tot['in8']:.4f}  coded plane "
              f"{ent['e5m2'] / nvals:.3f} bits/value")


if __name__ == "__main__":
    main()
