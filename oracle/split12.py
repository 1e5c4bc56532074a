"""Split12 weight format, stated plainly in numpy.

TEST INFRASTRUCTURE ONLY: the slow reference for a bf16 format read from the
"weight-compression" README (Split12: bf16 split into its two bytes, the high
byte rebuilt from a codebook, the low byte kept raw; 24.967 % smaller on a
753B model, i.e. 12 bits a value plus a little).  Only the tests, the smoke
check and the benchmark's CPU leg may import it; the CUDA library never does.

Reading (the page gives the idea, not the format):
  * high byte h = b >> 8 (sign and exponent bits 7..1), low byte l = b & 0xFF;
  * codebook: the K <= 16 most frequent high bytes of the tensor (ties to the
    smaller byte), stored in ascending order;
  * each value stores a 4-bit index into the codebook (value i in byte i // 2,
    low nibble when i is even; 0 for a value whose high byte is not in the
    codebook) and its low byte;
  * values whose high byte is not in the codebook are exceptions, listed per
    65,536-value chunk in ascending position: u16 position in the chunk and
    the u8 high byte; a u64 offset table gives each chunk's first exception.

Container (little-endian, sections 16-byte aligned, zero padding):
    0   "W12C"  u16 version 1  u8 dtype 1 (bf16)  u8 K (codebook entries)
    8   u64 n
    16  u32 chunk values 65536  u32 nc = ceil(n / 65536)
    24  u64 ne (exceptions)
    32  u64 off_idx   40 u64 off_lo   48 u64 off_exc   56 u64 total bytes
    64  u8 codebook[16] (entries >= K are 0)
    80  u64 exc_off[nc + 1]
    off_idx   ceil(n / 2) index bytes
    off_lo    n low bytes
    off_exc   u16 position[ne], then (16-aligned) u8 high byte[ne]
"""
from __future__ import annotations

import numpy as np

CHUNK = 65536
MAGIC = b"W12C"
HEADER = 64
BOOK = 16


def _r16(v: int) -> int:
    return (v + 15) // 16 * 16


def layout(n: int, ne: int) -> dict:
    nc = -(-n // CHUNK)
    off_excoff = HEADER + BOOK
    off_idx = _r16(off_excoff + 8 * (nc + 1))
    off_lo = _r16(off_idx + (n + 1) // 2)
    off_exc = _r16(off_lo + n)
    off_excval = off_exc + _r16(2 * ne)
    total = off_excval + _r16(ne)
    return dict(nc=nc, off_excoff=off_excoff, off_idx=off_idx, off_lo=off_lo,
                off_exc=off_exc, off_excval=off_excval, total=total)


def codebook(high: np.ndarray) -> np.ndarray:
    """The up to 16 most frequent bytes of `high` (ties to the smaller byte),
    ascending."""
    counts = np.bincount(high, minlength=256)
    ranked = sorted(range(256), key=lambda b: (-int(counts[b]), b))
    chosen = [b for b in ranked[:BOOK] if counts[b] > 0]
    return np.array(sorted(chosen), dtype=np.uint8)


def encode(bits: np.ndarray) -> np.ndarray:
    """Container bytes for bf16 bits (uint16)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16).reshape(-1)
    n = bits.size
    high = (bits >> 8).astype(np.uint8)
    low = (bits & 0xFF).astype(np.uint8)
    book = codebook(high)
    k = book.size
    where = np.full(256, -1, np.int64)
    where[book] = np.arange(k)
    slot = where[high]
    is_exc = slot < 0
    idx = np.where(is_exc, 0, slot).astype(np.uint8)
    pos = np.nonzero(is_exc)[0]                      # ascending
    ne = pos.size
    L = layout(n, ne)
    # exceptions before the start of each chunk, and at the end
    exc_off = np.searchsorted(pos, np.arange(L["nc"] + 1, dtype=np.int64) * CHUNK)
    exc_off[-1] = ne
    out = np.zeros(L["total"], np.uint8)
    out[0:4] = np.frombuffer(MAGIC, np.uint8)
    out[4:6] = np.array([1], "<u2").view(np.uint8)
    out[6] = 1
    out[7] = k
    out[8:16] = np.array([n], "<u8").view(np.uint8)
    out[16:24] = np.array([CHUNK, L["nc"]], "<u4").view(np.uint8)
    out[24:32] = np.array([ne], "<u8").view(np.uint8)
    out[32:64] = np.array([L["off_idx"], L["off_lo"], L["off_exc"], L["total"]], "<u8").view(np.uint8)
    out[HEADER:HEADER + k] = book
    o = L["off_excoff"]
    out[o:o + 8 * (L["nc"] + 1)] = exc_off.astype("<u8").view(np.uint8)
    padded = np.zeros(2 * ((n + 1) // 2), np.uint8)
    padded[:n] = idx
    out[L["off_idx"]:L["off_idx"] + padded.size // 2] = padded[0::2] | (padded[1::2] << 4)
    out[L["off_lo"]:L["off_lo"] + n] = low
    if ne:
        out[L["off_exc"]:L["off_exc"] + 2 * ne] = (pos % CHUNK).astype("<u2").view(np.uint8)
        out[L["off_excval"]:L["off_excval"] + ne] = high[pos]
    return out


def _u(c: np.ndarray, off: int, fmt: str) -> int:
    return int(np.frombuffer(c[off:off + np.dtype(fmt).itemsize].tobytes(), fmt)[0])


def read_header(cont: np.ndarray) -> dict:
    c = np.ascontiguousarray(cont, dtype=np.uint8)
    if c.size < HEADER + BOOK or c[:4].tobytes() != MAGIC or _u(c, 4, "<u2") != 1 or c[6] != 1:
        raise ValueError("not a Split12 container")
    n, ne = _u(c, 8, "<u8"), _u(c, 24, "<u8")
    k = int(c[7])
    L = layout(n, ne)
    if (_u(c, 16, "<u4") != CHUNK or _u(c, 20, "<u4") != L["nc"] or not 0 <= k <= BOOK
            or (n > 0) != (k > 0)):
        raise ValueError("bad Split12 header")
    if [_u(c, 32 + 8 * j, "<u8") for j in range(4)] != [L["off_idx"], L["off_lo"], L["off_exc"], L["total"]]:
        raise ValueError("bad Split12 layout")
    if c.size < L["total"]:
        raise ValueError("Split12 container cut short")
    return dict(n=n, ne=ne, k=k, **L)


def decode(cont: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) of a container.  Checks what decoding relies on:
    the header and layout, a non-decreasing exception table ending at ne,
    every index below K, and exception positions inside their chunk, inside
    n and ascending within the chunk (ValueError otherwise)."""
    c = np.ascontiguousarray(cont, dtype=np.uint8)
    h = read_header(c)
    n, ne, k, nc = h["n"], h["ne"], h["k"], h["nc"]
    book = c[HEADER:HEADER + BOOK]
    o = h["off_excoff"]
    exc_off = c[o:o + 8 * (nc + 1)].view("<u8").astype(np.int64)
    if exc_off[0] != 0 or exc_off[-1] != ne or np.any(np.diff(exc_off) < 0):
        raise ValueError("bad Split12 exception table")
    packed = c[h["off_idx"]:h["off_idx"] + (n + 1) // 2]
    idx = np.empty(2 * packed.size, np.uint8)
    idx[0::2] = packed & 0xF
    idx[1::2] = packed >> 4
    idx = idx[:n]
    if np.any(idx >= max(k, 1)):
        raise ValueError("codebook index out of range")
    low = c[h["off_lo"]:h["off_lo"] + n].astype(np.uint16)
    out = (book[idx].astype(np.uint16) << 8) | low
    for ch in range(nc):
        e0, e1 = int(exc_off[ch]), int(exc_off[ch + 1])
        if e0 == e1:
            continue
        p = c[h["off_exc"] + 2 * e0:h["off_exc"] + 2 * e1].view("<u2").astype(np.int64)
        if np.any(np.diff(p) <= 0) or ch * CHUNK + p[-1] >= n:
            raise ValueError("bad Split12 exception position")
        val = c[h["off_excval"] + e0:h["off_excval"] + e1].astype(np.uint16)
        i = ch * CHUNK + p
        out[i] = (val << 8) | low[i]
    return out


def canonical(cont: np.ndarray) -> bool:
    """Whether a decodable container is the one that encode() writes for its
    values: codebook ascending, zero-padded and equal to the values' 16 most
    frequent high bytes; every exception marked by index 0 and missing from
    the codebook; padding zero."""
    c = np.ascontiguousarray(cont, dtype=np.uint8)
    vals = decode(c)
    return c.size == read_header(c)["total"] and np.array_equal(encode(vals), c)


def linear(x_bits: np.ndarray, cont: np.ndarray, n_rows: int) -> np.ndarray:
    """Y = X W^T in float64, W (n_rows x K, bf16) decoded from a container and
    X (M x K) given as bf16 bits: the exact products of the bf16 values,
    summed in float64 (the reference a fused decode-and-multiply kernel is
    held to within its fp32 accumulation bound)."""
    w = decode(cont)
    k = w.size // n_rows
    if n_rows * k != w.size:
        raise ValueError("container size is not a multiple of the row count")
    to_f = lambda b: (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    wf = to_f(w).astype(np.float64).reshape(n_rows, k)
    xf = to_f(x_bits).astype(np.float64).reshape(-1, k)
    return xf @ wf.T
