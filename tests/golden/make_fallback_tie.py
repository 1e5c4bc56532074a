"""Writes the two raw-fallback boundary fixtures under tests/golden/:

  container_bf16_n186_tie_raw.txt     128 + 2w == nsym: stored raw
  container_bf16_n186_near_coded.txt  128 + 2w == nsym - 2: kept coded

The rule they pin ("PTWM", Configuration table, compression_threshold: data
whose coded form does not shrink is stored as it is) is read as: a chunk is
stored raw iff its coded length 128 + 2w is >= nsym, so a tie goes raw.

Each input is 186 bf16 values with zero sign and mantissa (value bits =
exponent << 7), exponents drawn uniformly from 120..127 by numpy PCG64 with
the seed given below; the two seeds were found by searching for the two
word counts.  Only the oracle's pinned pieces are called -- histogram,
normalize and the rANS core (pinned by the worked traces and brute force) --
to get the table and w; the container bytes are laid out here, field by
field, from the container description, not by the oracle's encoder.

    python tests/golden/make_fallback_tie.py
"""
from __future__ import annotations

import os
import struct
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(os.path.dirname(os.path.dirname(HERE)), "oracle"))
import oracle  # noqa: E402

N = 186
CASES = (("container_bf16_n186_tie_raw.txt", 161, 29, "raw"),
         ("container_bf16_n186_near_coded.txt", 68, 28, "coded"))


def exponents(seed: int) -> np.ndarray:
    rng = np.random.default_rng([7, N, seed])
    rng.integers(2, 9)  # the search drew the alphabet size first (8 here)
    return (120 + rng.integers(0, 8, N)).astype(np.uint8)


def r16(v: int) -> int:
    return (v + 15) & ~15


def container(e: np.ndarray, freq: np.ndarray, states, words, raw: bool) -> bytes:
    n = e.size
    off_choff, off_chlen = 576, 576 + 16
    off_raw = r16(off_chlen + 4)
    off_exp = r16(off_raw + n)
    if raw:
        payload = e.tobytes()
    else:
        payload = np.asarray(states, "<u4").tobytes() + np.asarray(words, "<u2").tobytes()
    exp_bytes = r16(len(payload))
    total = off_exp + exp_bytes
    buf = bytearray(total)
    buf[0:64] = (b"WCZ1" + struct.pack("<HBB", 1, 1, 32) + struct.pack("<Q", n) +
                 struct.pack("<II", 65536, 1) + struct.pack("<HHI", 12, 0, 0) +
                 struct.pack("<QQQQ", off_raw, off_exp, exp_bytes, total))
    buf[64:576] = np.asarray(freq, "<u2").tobytes()
    buf[off_choff:off_choff + 16] = struct.pack("<QQ", 0, exp_bytes)
    buf[off_chlen:off_chlen + 4] = struct.pack("<I", len(payload))
    # raw plane: sign + mantissa bytes, all zero for these values
    buf[off_exp:off_exp + len(payload)] = payload
    return bytes(buf)


def write(fname: str, seed: int, e: np.ndarray, freq, w: int, decision: str, data: bytes):
    lines = [
        f"# Raw-fallback boundary: {N} bf16 values, bits = exponent << 7 (sign and",
        f"# mantissa zero); exponents 120..127 from PCG64([7, {N}, {seed}]).",
        "# Table (histogram -> 12-bit normalisation): " +
        ", ".join(f"{s}:{int(freq[s])}" for s in range(256) if freq[s]),
        f"# rANS core: w = {w} words -> coded length 128 + 2w = {128 + 2 * w}, nsym = {N}",
        f"# decision: {decision} (raw iff 128 + 2w >= nsym)",
        "# Written by tests/golden/make_fallback_tie.py.",
        "# Format: '<offset>: <hex bytes>'; bytes not listed are 0x00; 'exponents:'",
        "# lists the input's exponent bytes.",
        "exponents: " + " ".join(f"{int(x):02x}" for x in e),
        f"length: {len(data)}",
    ]
    for off in range(0, len(data), 16):
        row = data[off:off + 16]
        if any(row):
            lines.append(f"{off}: " + " ".join(f"{b:02x}" for b in row))
    with open(os.path.join(HERE, fname), "w") as fh:
        fh.write("\n".join(lines) + "\n")


def main():
    for fname, seed, want_w, decision in CASES:
        e = exponents(seed)
        freq = oracle.normalize(oracle.histogram(e))
        states, words = oracle.rans_encode(e, freq)
        w = int(words.size)
        assert w == want_w, (fname, w)
        raw = 128 + 2 * w >= N
        assert raw == (decision == "raw")
        write(fname, seed, e, freq, w, decision, container(e, freq, states, words, raw))


if __name__ == "__main__":
    main()
