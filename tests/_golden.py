"""Readers for the hand-worked fixtures under tests/golden/."""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ints(field: str) -> list[int]:
    out: list[int] = []
    if not field:
        return out
    for tok in field.split(","):
        if "*" in tok:
            v, c = tok.split("*")
            out.extend([int(v, 0)] * int(c))
        else:
            out.append(int(tok, 0))
    return out


def load_traces() -> dict:
    traces = {}
    with open(os.path.join(GOLDEN, "rans_traces.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, *fields = line.split()
            kv = dict(f.split("=", 1) for f in fields)
            freq = np.zeros(256, np.uint16)
            for item in kv["freq"].split(","):
                s, f = item.split(":")
                freq[int(s)] = int(f)
            traces[name] = dict(
                lanes=int(kv["lanes"]),
                freq=freq,
                syms=np.array(_ints(kv["syms"]), np.uint8),
                states=_ints(kv["states"]),
                words=_ints(kv["words"]),
            )
    return traces


def load_container(fname: str) -> np.ndarray:
    data = None
    with open(os.path.join(GOLDEN, fname)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            if not key[0].isdigit() and key != "length":
                continue  # a named field (load_fields)
            if key == "length":
                data = np.zeros(int(val), np.uint8)
                continue
            bs = [int(b, 16) for b in val.split()]
            if "*" in key:
                off, cnt = (int(x) for x in key.split("*"))
            else:
                off, cnt = int(key), 1
            for r in range(cnt):
                data[off + r * len(bs): off + (r + 1) * len(bs)] = bs
    return data


def load_fields(fname: str) -> dict:
    """The named (non-offset) fields of a fixture, e.g. 'exponents', as byte
    lists parsed from hex."""
    out = {}
    with open(os.path.join(GOLDEN, fname)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            if key[0].isdigit() or key == "length":
                continue
            out[key] = [int(b, 16) for b in val.split()]
    return out
