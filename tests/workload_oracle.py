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


def oracle_chunk_payloads(args):
    """Payload bytes (as stored in the container) of a few chunks of one
    tensor, computed with the oracle's rANS core and the whole tensor's table."""
    cid, idx, chunks = args
    import numpy as np
    import oracle
    import workloads
    bits = workloads.generate_tensor(cid, idx)
    if bits.dtype == np.uint16:
        e, _ = oracle.split_bf16(bits)
    else:
        e, _, _ = oracle.split_fp32(bits)
    f = oracle.normalize(oracle.histogram(e))
    out = {}
    for k in chunks:
        sym = e[k * 65536:(k + 1) * 65536]
        states, words = oracle.rans_encode(sym, f)
        if 128 + 2 * words.size < sym.size:
            payload = states.astype("<u4").tobytes() + words.astype("<u2").tobytes()
        else:
            payload = sym.tobytes()
        out[k] = hashlib.sha256(payload).hexdigest()
    return idx, f.tobytes(), out


def gen_tensor(args):
    cid, idx = args
    import workloads
    return idx, workloads.generate_tensor(cid, idx)
