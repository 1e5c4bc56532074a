"""Worker-side helpers for the full-size workload tests: each call regenerates
one seeded tensor and returns the digest of the CPU oracle's container (so
that no tensor data crosses process boundaries).  Run in spawn-started pools."""
from __future__ import annotations

import hashlib
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, os.path.join(ROOT, "oracle")):
    if p not in sys.path:
        sys.path.insert(0, p)


def oracle_digest(args):
    cid, idx = args
    import oracle
    import workloads
    bits = workloads.generate_tensor(cid, idx)
    cont = oracle.encode(bits)
    return idx, cont.size, hashlib.sha256(cont.tobytes()).hexdigest()


def gen_tensor_and_digest(args):
    """The tensor and the digest of the oracle's container for it, from one
    draw."""
    cid, idx = args
    import oracle
    import workloads
    bits = workloads.generate_tensor(cid, idx)
    cont = oracle.encode(bits)
    return idx, bits, cont.size, hashlib.sha256(cont.tobytes()).hexdigest()


def gen_tensor(args):
    cid, idx = args
    import workloads
    return idx, workloads.generate_tensor(cid, idx)
