"""Seeded synthetic weight tensors for the five workloads.

This module only draws inputs; it holds none of the codec's arithmetic.  Both
the CPU oracle (tests, CPU baseline) and the CUDA library (tests, benchmark)
take their inputs from here.  Real checkpoints are not available, so every
tensor is drawn from numpy's PCG64 generator with a fixed seed, in the shapes
of the models the pages measure on (GPT-2 small in "SMEF -- blog companion
code"; bf16 decoder LMs in "weight-compression" and "seedpack"):

  1  one bf16 1024x1024 tensor, N(0, 0.02) drawn in fp32, seed 0.
  2  bf16 tensor set shaped like a 0.6B decoder LM (hidden 1024, 28 layers):
     per layer q 1024x2048, k 1024x1024, v 1024x1024, o 2048x1024,
     gate 1024x3072, up 1024x3072, down 3072x1024, drawn N(0, 0.02/sqrt(l+1))
     with l the 0-based layer; then the 151936x1024 embedding, N(0, 0.02);
     then 57 norm vectors of 1024 (two per layer and a final one),
     N(1.0, 0.05).
  3  fp32 tensor set shaped like GPT-2 small: 12 layers of 768x2304,
     768x768, 768x3072, 3072x768, then the 50257x768 embedding; N(0, 0.02).
  4  bf16 tensor set shaped like an 8B dense LM (hidden 4096, 32 layers, GQA):
     per layer q 4096x4096, k 4096x1024, v 4096x1024, o 4096x4096,
     gate 4096x14336, up 4096x14336, down 14336x4096; then the 128256x4096
     embedding; values 0.015 * Student-t with 4 degrees of freedom.
  5  one adversarial bf16 tensor of 2^28 values in 4096 chunks of 65536;
     chunk k is of kind k mod 4: (a) uniform random 16-bit patterns,
     (b) one random 16-bit pattern repeated, (c) a uniform mix of +-0,
     subnormals, +-Inf and NaNs with random non-zero payloads,
     (d) N(0, 1e-3).

Tensor i of workload c uses PCG64([c, i]) (workload 1: PCG64(0)).  fp32
samples become bf16 by round-to-nearest-even on the bits,
(u + 0x7FFF + ((u >> 16) & 1)) >> 16; the samplers give no NaN or Inf.
Student-t(4) is drawn as Z / sqrt(G / 2) with Z ~ N(0, 1) and G ~ Gamma(2, 1)
(so that 2G ~ chi-square with 4 degrees of freedom).
Arrays are returned as raw bits: uint16 for bf16, uint32 for fp32.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass

import numpy as np

CHUNK = 65536


@dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: tuple
    dtype: str          # "bf16" | "fp32"
    dist: str           # "normal" | "student_t4" | "adversarial"
    loc: float
    scale: float

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape))

    @property
    def itemsize(self) -> int:
        return 2 if self.dtype == "bf16" else 4


def _lm_layers(layers, shapes, dtype, dist, scale_fn):
    out = []
    for l in range(layers):
        for nm, shp in shapes:
            out.append(TensorSpec(f"layers.{l}.{nm}", shp, dtype, dist, 0.0, scale_fn(l)))
    return out


def tensor_specs(cid: int) -> list[TensorSpec]:
    if cid == 1:
        return [TensorSpec("w", (1024, 1024), "bf16", "normal", 0.0, 0.02)]
    if cid == 2:
        shapes = [("q", (1024, 2048)), ("k", (1024, 1024)), ("v", (1024, 1024)),
                  ("o", (2048, 1024)), ("gate", (1024, 3072)), ("up", (1024, 3072)),
                  ("down", (3072, 1024))]
        specs = _lm_layers(28, shapes, "bf16", "normal", lambda l: 0.02 / math.sqrt(l + 1))
        specs.append(TensorSpec("embed", (151936, 1024), "bf16", "normal", 0.0, 0.02))
        for l in range(28):
            specs.append(TensorSpec(f"layers.{l}.input_norm", (1024,), "bf16", "normal", 1.0, 0.05))
            specs.append(TensorSpec(f"layers.{l}.post_norm", (1024,), "bf16", "normal", 1.0, 0.05))
        specs.append(TensorSpec("final_norm", (1024,), "bf16", "normal", 1.0, 0.05))
        return specs
    if cid == 3:
        shapes = [("qkv", (768, 2304)), ("proj", (768, 768)), ("fc", (768, 3072)),
                  ("fc_proj", (3072, 768))]
        specs = _lm_layers(12, shapes, "fp32", "normal", lambda l: 0.02)
        specs.append(TensorSpec("wte", (50257, 768), "fp32", "normal", 0.0, 0.02))
        return specs
    if cid == 4:
        shapes = [("q", (4096, 4096)), ("k", (4096, 1024)), ("v", (4096, 1024)),
                  ("o", (4096, 4096)), ("gate", (4096, 14336)), ("up", (4096, 14336)),
                  ("down", (14336, 4096))]
        specs = _lm_layers(32, shapes, "bf16", "student_t4", lambda l: 0.015)
        specs.append(TensorSpec("embed", (128256, 4096), "bf16", "student_t4", 0.0, 0.015))
        return specs
    if cid == 5:
        return [TensorSpec("adversarial", (1 << 28,), "bf16", "adversarial", 0.0, 0.0)]
    raise ValueError(f"no workload {cid}")


def rne_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _rng(cid: int, idx: int) -> np.random.Generator:
    if cid == 1:
        return np.random.Generator(np.random.PCG64(0))
    return np.random.Generator(np.random.PCG64([cid, idx]))


def _adversarial_chunks(rng: np.random.Generator, nchunks: int, first_chunk: int = 0) -> np.ndarray:
    """Chunk k (absolute index first_chunk + j) is of kind k mod 4."""
    out = np.empty((nchunks, CHUNK), np.uint16)
    kinds = (np.arange(nchunks) + first_chunk) % 4
    ia, ib, ic, id_ = (np.nonzero(kinds == q)[0] for q in range(4))
    if ia.size:
        out[ia] = rng.integers(0, 1 << 16, size=(ia.size, CHUNK), dtype=np.uint16)
    if ib.size:
        pat = rng.integers(0, 1 << 16, size=ib.size, dtype=np.uint16)
        out[ib] = pat[:, None]
    if ic.size:
        cls = rng.integers(0, 4, size=(ic.size, CHUNK), dtype=np.uint8)
        sign = rng.integers(0, 2, size=(ic.size, CHUNK), dtype=np.uint16) << np.uint16(15)
        mant = rng.integers(1, 128, size=(ic.size, CHUNK), dtype=np.uint16)
        v = np.where(cls == 0, sign,
            np.where(cls == 1, sign | mant,
            np.where(cls == 2, sign | np.uint16(0x7F80), sign | np.uint16(0x7F80) | mant)))
        out[ic] = v.astype(np.uint16)
    if id_.size:
        out[id_] = rne_bf16(rng.standard_normal((id_.size, CHUNK), dtype=np.float32)
                            * np.float32(1e-3))
    return out.reshape(-1)


def adversarial_kind_tensor(kind: int, nchunks: int, seed: int = 0) -> np.ndarray:
    """A standalone tensor made only of chunks of one adversarial kind
    (0=a, 1=b, 2=c, 3=d), so that kind (b) gets a single-symbol table."""
    rng = np.random.Generator(np.random.PCG64([5, 1000 + 10 * kind + seed]))
    full = _adversarial_chunks(rng, nchunks * 4, first_chunk=0).reshape(nchunks * 4, CHUNK)
    return np.ascontiguousarray(full[kind::4][:nchunks]).reshape(-1)


def generate(spec: TensorSpec, cid: int, idx: int) -> np.ndarray:
    rng = _rng(cid, idx)
    n = spec.numel
    if spec.dist == "adversarial":
        return _adversarial_chunks(rng, n // CHUNK)
    if spec.dist == "normal":
        x = rng.standard_normal(n, dtype=np.float32)
        x *= np.float32(spec.scale)
        if spec.loc:
            x += np.float32(spec.loc)
    elif spec.dist == "student_t4":
        z = rng.standard_normal(n, dtype=np.float32)
        g = rng.standard_gamma(2.0, size=n, dtype=np.float32)
        g *= np.float32(0.5)
        np.sqrt(g, out=g)
        z /= g
        z *= np.float32(spec.scale)
        x = z
    else:
        raise ValueError(spec.dist)
    if spec.dtype == "bf16":
        return rne_bf16(x)
    return x.view(np.uint32)


def generate_tensor(cid: int, idx: int) -> np.ndarray:
    return generate(tensor_specs(cid)[idx], cid, idx)


def _worker(args):
    cid, idx = args
    return idx, generate_tensor(cid, idx)


def generate_config(cid: int, indices=None, workers: int | None = None) -> list[np.ndarray]:
    """All (or the listed) tensors of a workload, in order.  workers > 1 draws
    tensors in a spawn-started process pool (each tensor keeps its own seed,
    so the result does not depend on the worker count)."""
    specs = tensor_specs(cid)
    if indices is None:
        indices = list(range(len(specs)))
    if workers is None:
        workers = 1
    if workers <= 1 or len(indices) <= 1:
        return [generate_tensor(cid, i) for i in indices]
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = {}
    with ctx.Pool(min(workers, len(indices))) as pool:
        for idx, arr in pool.imap_unordered(_worker, [(cid, i) for i in indices]):
            out[idx] = arr
    return [out[i] for i in indices]


def default_workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)
