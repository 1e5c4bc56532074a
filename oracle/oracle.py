"""ctypes wrapper around the CPU oracle (wc_oracle.c).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain scalar statement of the
exponent-plane rANS container; only the tests, the smoke check and the
CPU-baseline leg of the benchmark may import this module.  The CUDA library
never calls it and shares no code with it.

Pins of every oracle function (worked traces, normalisation examples, brute
force, the rANS accounting bound, exhaustive bf16 round trip, fp32 special
values, CRC-32 check values and zlib) live in tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wc_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

OK, ERR_INVALID_ARG, ERR_CAPACITY, ERR_CORRUPT = 0, 1, 2, 4
BF16, FP32, FP16, FP8E4M3, FP8E5M2, BF16_HIGHBYTE = 1, 2, 3, 4, 5, 6
_NP = {BF16: np.uint16, FP32: np.uint32, FP16: np.uint16, FP8E4M3: np.uint8,
       FP8E5M2: np.uint8, BF16_HIGHBYTE: np.uint16}
CHUNK = 65536


def build(force: bool = False) -> str:
    """Compile wc_oracle.c into liboracle.so (plain -O2, single thread)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "wc_oracle.h"))
    ):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-shared", "-fPIC",
             SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        vp = ctypes.c_void_p
        L.oracle_encode_bound.restype = ctypes.c_uint64
        L.oracle_encode_bound.argtypes = [ctypes.c_uint64, ctypes.c_int]
        L.oracle_split_bf16.argtypes = [vp, ctypes.c_uint64, vp, vp]
        L.oracle_split_fp32.argtypes = [vp, ctypes.c_uint64, vp, vp, vp]
        L.oracle_split_fp16.argtypes = [vp, ctypes.c_uint64, vp, vp]
        L.oracle_split_fp8e4m3.argtypes = [vp, ctypes.c_uint64, vp, vp]
        L.oracle_split_fp8e5m2.argtypes = [vp, ctypes.c_uint64, vp, vp]
        L.oracle_split_bf16_highbyte.argtypes = [vp, ctypes.c_uint64, vp, vp]
        L.oracle_histogram.argtypes = [vp, ctypes.c_uint64, vp]
        L.oracle_normalize.argtypes = [vp, vp]
        L.oracle_rans_encode.argtypes = [vp, ctypes.c_uint32, vp, ctypes.c_uint32, vp, vp, u32p]
        L.oracle_rans_decode.argtypes = [vp, vp, ctypes.c_uint32, ctypes.c_uint32, vp,
                                         ctypes.c_uint32, vp]
        L.oracle_encode.argtypes = [vp, ctypes.c_uint64, ctypes.c_int, vp, ctypes.c_uint64, u64p]
        L.oracle_decode.argtypes = [vp, ctypes.c_uint64, vp, ctypes.c_uint64]
        L.oracle_decode_chunk.argtypes = [vp, ctypes.c_uint64, ctypes.c_uint64, vp, ctypes.c_uint64]
        L.oracle_read_header.argtypes = [vp, ctypes.c_uint64, u64p, ctypes.POINTER(ctypes.c_int), u64p]
        L.oracle_chunk_accounting.argtypes = [vp, ctypes.c_uint32, vp,
                                              ctypes.POINTER(ctypes.c_double),
                                              ctypes.POINTER(ctypes.c_double),
                                              ctypes.POINTER(ctypes.c_double)]
        L.oracle_crc32.restype = ctypes.c_uint32
        L.oracle_crc32.argtypes = [vp, ctypes.c_uint64]
        L.oracle_crc32_blocks.argtypes = [vp, ctypes.c_uint64, ctypes.c_uint64, vp]
        del u8p, u16p, u64p
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def dtype_code(arr: np.ndarray) -> int:
    if arr.dtype == np.uint16:
        return BF16
    if arr.dtype == np.uint32:
        return FP32
    if arr.dtype == np.float16:
        return FP16
    if arr.dtype == np.uint8:
        return FP8E4M3
    raise TypeError("oracle takes bf16 bits as uint16, fp32 bits as uint32, fp16 as float16, "
                    "fp8 e4m3 bits as uint8")


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: oracle status {code}")
        self.code = code


def encode_bound(n: int, dtype: int) -> int:
    return int(lib().oracle_encode_bound(n, dtype))


def split_bf16(bits: np.ndarray):
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    n = bits.size
    e = np.empty(n, np.uint8)
    sm = np.empty(n, np.uint8)
    lib().oracle_split_bf16(_ptr(bits), n, _ptr(e), _ptr(sm))
    return e, sm


def split_fp16(bits: np.ndarray):
    """(coded high-byte plane, raw low-byte plane) of fp16 bits (uint16)."""
    bits = np.ascontiguousarray(bits).view(np.uint16).reshape(-1)
    hi = np.zeros(bits.size, np.uint8)
    lo = np.zeros(bits.size, np.uint8)
    lib().oracle_split_fp16(_ptr(bits), bits.size, _ptr(hi), _ptr(lo))
    return hi, lo


def split_fp8e4m3(bits: np.ndarray):
    """(exponent-nibble plane, packed low-nibble plane) of fp8 e4m3 bits (uint8)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8).reshape(-1)
    e = np.zeros(bits.size, np.uint8)
    nib = np.zeros((bits.size + 1) // 2, np.uint8)
    lib().oracle_split_fp8e4m3(_ptr(bits), bits.size, _ptr(e), _ptr(nib) if nib.size else None)
    return e, nib


def split_fp8e5m2(bits: np.ndarray):
    """(high-nibble plane, packed low-nibble plane) of fp8 e5m2 bits (uint8)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8).reshape(-1)
    hi = np.zeros(bits.size, np.uint8)
    nib = np.zeros((bits.size + 1) // 2, np.uint8)
    lib().oracle_split_fp8e5m2(_ptr(bits), bits.size, _ptr(hi), _ptr(nib) if nib.size else None)
    return hi, nib


def split_bf16_highbyte(bits: np.ndarray):
    """(high-byte plane, low-byte plane) of bf16 bits (uint16), no reorder."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16).reshape(-1)
    hi = np.zeros(bits.size, np.uint8)
    lo = np.zeros(bits.size, np.uint8)
    lib().oracle_split_bf16_highbyte(_ptr(bits), bits.size, _ptr(hi), _ptr(lo))
    return hi, lo


def split_fp32(bits: np.ndarray):
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    n = bits.size
    e = np.empty(n, np.uint8)
    sign = np.zeros((n + 7) // 8, np.uint8)
    mant = np.empty(3 * n, np.uint8)
    lib().oracle_split_fp32(_ptr(bits), n, _ptr(e), _ptr(sign) if sign.size else None,
                            _ptr(mant) if mant.size else None)
    return e, sign, mant


def histogram(e: np.ndarray) -> np.ndarray:
    e = np.ascontiguousarray(e, dtype=np.uint8)
    c = np.zeros(256, np.uint64)
    lib().oracle_histogram(_ptr(e) if e.size else None, e.size, _ptr(c))
    return c


def normalize(counts) -> np.ndarray:
    c = np.zeros(256, np.uint64)
    if isinstance(counts, dict):
        for s, v in counts.items():
            c[s] = v
    else:
        c[:] = np.asarray(counts, dtype=np.uint64)
    f = np.zeros(256, np.uint16)
    st = lib().oracle_normalize(_ptr(c), _ptr(f))
    if st:
        raise OracleError(st, "normalize")
    return f


def rans_encode(sym, freq, lanes: int = 32):
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    freq = np.ascontiguousarray(freq, dtype=np.uint16)
    assert freq.size == 256
    states = np.zeros(lanes, np.uint32)
    words = np.zeros(max(sym.size, 1), np.uint16)
    w = ctypes.c_uint32(0)
    st = lib().oracle_rans_encode(_ptr(sym), sym.size, _ptr(freq), lanes, _ptr(states),
                                  _ptr(words), ctypes.byref(w))
    if st:
        raise OracleError(st, "rans_encode")
    return states, words[: w.value].copy()


def rans_decode(states, words, nsym: int, freq, lanes: int = 32):
    states = np.ascontiguousarray(states, dtype=np.uint32)
    words = np.ascontiguousarray(words, dtype=np.uint16)
    if words.size == 0:
        words = np.zeros(1, np.uint16)[:0].copy()
    freq = np.ascontiguousarray(freq, dtype=np.uint16)
    out = np.zeros(max(nsym, 1), np.uint8)
    wbuf = words if words.size else np.zeros(1, np.uint16)
    st = lib().oracle_rans_decode(_ptr(states), _ptr(wbuf), words.size, nsym, _ptr(freq),
                                  lanes, _ptr(out))
    return st, out[:nsym]


def encode(bits: np.ndarray, dtype: int | None = None) -> np.ndarray:
    """Container bytes for a flat array of bf16 (uint16) or fp32 (uint32) bits,
    fp16 values (float16, or uint16 bits with dtype=FP16), fp8 bits (uint8:
    e4m3 unless dtype=FP8E5M2), or bf16 bits with dtype=BF16_HIGHBYTE."""
    bits = np.ascontiguousarray(bits).reshape(-1)
    dt = dtype_code(bits) if dtype is None else dtype
    if dt == FP16:
        bits = bits.view(np.uint16)
    n = bits.size
    cap = encode_bound(n, dt)
    out = np.empty(cap, np.uint8)
    size = ctypes.c_uint64(0)
    st = lib().oracle_encode(_ptr(bits) if n else None, n, dt, _ptr(out), cap, ctypes.byref(size))
    if st:
        raise OracleError(st, "encode")
    return out[: size.value].copy()


def read_header(cont: np.ndarray):
    cont = np.ascontiguousarray(cont, dtype=np.uint8)
    n = ctypes.c_uint64(0)
    dt = ctypes.c_int(0)
    nc = ctypes.c_uint64(0)
    st = lib().oracle_read_header(_ptr(cont), cont.size, ctypes.byref(n), ctypes.byref(dt),
                                  ctypes.byref(nc))
    if st:
        raise OracleError(st, "read_header")
    return n.value, dt.value, nc.value


def decode_status(cont: np.ndarray, n_hint: int | None = None, dtype_hint: int | None = None):
    """(status, values) without raising; values is None when the header is bad."""
    cont = np.ascontiguousarray(cont, dtype=np.uint8)
    n = ctypes.c_uint64(0)
    dt = ctypes.c_int(0)
    nc = ctypes.c_uint64(0)
    st = lib().oracle_read_header(_ptr(cont), cont.size, ctypes.byref(n), ctypes.byref(dt),
                                  ctypes.byref(nc))
    if st:
        return st, None
    npdt = _NP[dt.value]
    out = np.zeros(max(n.value, 1), npdt)
    st = lib().oracle_decode(_ptr(cont), cont.size, _ptr(out), out.nbytes)
    return st, out[: n.value]


def decode(cont: np.ndarray) -> np.ndarray:
    st, out = decode_status(cont)
    if st:
        raise OracleError(st, "decode")
    return out


def decode_chunk(cont: np.ndarray, k: int) -> np.ndarray:
    cont = np.ascontiguousarray(cont, dtype=np.uint8)
    n, dt, nc = read_header(cont)
    npdt = _NP[dt]
    nsym = min(CHUNK, n - k * CHUNK) if k < nc else 0
    out = np.zeros(max(nsym, 1), npdt)
    st = lib().oracle_decode_chunk(_ptr(cont), cont.size, k, _ptr(out), out.nbytes)
    if st:
        raise OracleError(st, "decode_chunk")
    return out[:nsym]


def chunk_accounting(sym, freq):
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    freq = np.ascontiguousarray(freq, dtype=np.uint16)
    a, b, c = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    st = lib().oracle_chunk_accounting(_ptr(sym), sym.size, _ptr(freq), ctypes.byref(a),
                                       ctypes.byref(b), ctypes.byref(c))
    if st:
        raise OracleError(st, "chunk_accounting")
    return a.value, b.value, c.value


def _bytes_view(data) -> np.ndarray:
    if isinstance(data, (bytes, bytearray, memoryview)):
        return np.frombuffer(bytes(data), dtype=np.uint8)
    return np.ascontiguousarray(data).reshape(-1).view(np.uint8)


def crc32(data) -> int:
    """CRC-32 (zlib / IEEE 802.3) of a byte string or array's bytes."""
    buf = _bytes_view(data)
    return int(lib().oracle_crc32(_ptr(buf) if buf.size else None, buf.size))


def crc32_blocks(data, block_bytes: int) -> np.ndarray:
    """CRC-32 of each block_bytes-sized block (the last one may be shorter)."""
    buf = _bytes_view(data)
    nb = -(-buf.size // block_bytes) if block_bytes > 0 else 0
    out = np.zeros(nb, dtype=np.uint32)
    st = lib().oracle_crc32_blocks(_ptr(buf) if buf.size else None, buf.size, block_bytes,
                                   _ptr(out) if nb else None)
    if st != OK:
        raise OracleError(st, "oracle_crc32_blocks")
    return out
