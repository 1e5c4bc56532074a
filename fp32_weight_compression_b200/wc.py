"""Python binding of libwc.so (include/wc.h): argument marshalling only.

Every step of encoding and decoding runs in the library's CUDA kernels; this
module only allocates device buffers through PyTorch, passes pointers, sizes
and the current stream, and turns status codes into exceptions.  There is no
CPU path: if libwc.so is missing or no CUDA device is present the calls fail.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwc.so")

OK, ERR_INVALID_ARG, ERR_CAPACITY, ERR_CUDA, ERR_CORRUPT, ERR_UNSUPPORTED, ERR_TIMEOUT = 0, 1, 2, 3, 4, 5, 6
BF16, FP32, FP16, FP8E4M3, FP8E5M2 = 1, 2, 3, 4, 5
CHUNK = 65536

_DT = {torch.bfloat16: BF16, torch.float32: FP32, torch.float16: FP16,
       torch.float8_e4m3fn: FP8E4M3, torch.float8_e5m2: FP8E5M2}
_TORCH_DT = {BF16: torch.bfloat16, FP32: torch.float32, FP16: torch.float16,
             FP8E4M3: torch.float8_e4m3fn, FP8E5M2: torch.float8_e5m2}
_ELEM = {BF16: 2, FP32: 4, FP16: 2, FP8E4M3: 1, FP8E5M2: 1}

EXPORTS = (
    "wc_encode_bound", "wc_scratch_bytes", "wc_encode", "wc_decode", "wc_decode_chunk",
    "wc_read_header", "wc_encode_batch", "wc_decode_batch", "wc_status_string", "wc_last_error",
    "wc_encode_noalloc", "wc_host_encode_footprint", "wc_host_decode_footprint", "wc_host_plan",
    "wc_encode_host", "wc_decode_host",
)
# Library-held scratch of wc_encode_noalloc (WC_NOALLOC_SCRATCH_BYTES in wc.h).
NOALLOC_SCRATCH_BYTES = 16 << 20


class EncodeItem(ctypes.Structure):
    _fields_ = [("in_", ctypes.c_void_p), ("n", ctypes.c_uint64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("out", ctypes.c_void_p), ("out_cap", ctypes.c_uint64),
                ("scratch", ctypes.c_void_p), ("scratch_cap", ctypes.c_uint64),
                ("out_size", ctypes.c_void_p)]


class Split12EncodeItem(ctypes.Structure):
    _fields_ = [("in_", ctypes.c_void_p), ("n", ctypes.c_uint64), ("out", ctypes.c_void_p),
                ("out_cap", ctypes.c_uint64), ("scratch", ctypes.c_void_p), ("scratch_cap", ctypes.c_uint64),
                ("out_size", ctypes.c_void_p)]


class Split12DecodeItem(ctypes.Structure):
    _fields_ = [("cont", ctypes.c_void_p), ("cont_bytes", ctypes.c_uint64), ("out", ctypes.c_void_p),
                ("n", ctypes.c_uint64)]


class DecodeItem(ctypes.Structure):
    _fields_ = [("cont", ctypes.c_void_p), ("cont_bytes", ctypes.c_uint64),
                ("out", ctypes.c_void_p), ("out_cap", ctypes.c_uint64)]


class HostEncodeItem(ctypes.Structure):
    _fields_ = [("h_in", ctypes.c_void_p), ("n", ctypes.c_uint64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("h_out", ctypes.c_void_p), ("h_out_cap", ctypes.c_uint64),
                ("h_out_size", ctypes.c_void_p)]


class HostDecodeItem(ctypes.Structure):
    _fields_ = [("h_cont", ctypes.c_void_p), ("cont_bytes", ctypes.c_uint64),
                ("h_out", ctypes.c_void_p), ("out_cap", ctypes.c_uint64)]


class WCError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)}"
                         + (f" ({last_error()})" if code == ERR_CUDA else ""))
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libwc.so from this package directory (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m fp32_weight_compression_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    u64, i32, u32, vp = ctypes.c_uint64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p
    L.wc_encode_bound.restype = u64
    L.wc_encode_bound.argtypes = [u64, i32]
    L.wc_scratch_bytes.restype = u64
    L.wc_scratch_bytes.argtypes = [u64, i32]
    L.wc_encode.restype = i32
    L.wc_encode.argtypes = [vp, u64, i32, vp, u64, vp, u64, vp, vp]
    L.wc_decode.restype = i32
    L.wc_decode.argtypes = [vp, u64, vp, u64, vp, vp]
    L.wc_decode_chunk.restype = i32
    L.wc_decode_chunk.argtypes = [vp, u64, u64, vp, u64, vp, vp]
    L.wc_read_header.restype = i32
    L.wc_read_header.argtypes = [vp, u64, ctypes.POINTER(u64), ctypes.POINTER(i32), ctypes.POINTER(u64)]
    L.wc_encode_batch.restype = i32
    L.wc_encode_batch.argtypes = [ctypes.POINTER(EncodeItem), u32, vp]
    L.wc_decode_batch.restype = i32
    L.wc_decode_batch.argtypes = [ctypes.POINTER(DecodeItem), u32, vp, vp]
    L.wc_status_string.restype = ctypes.c_char_p
    L.wc_status_string.argtypes = [i32]
    L.wc_last_error.restype = ctypes.c_char_p
    L.wc_last_error.argtypes = []
    L.wc_encode_noalloc.restype = i32
    L.wc_encode_noalloc.argtypes = [vp, u64, i32, vp, u64, vp, vp]
    L.wc_host_encode_footprint.restype = u64
    L.wc_host_encode_footprint.argtypes = [u64, i32]
    L.wc_host_decode_footprint.restype = u64
    L.wc_host_decode_footprint.argtypes = [u64, u64, i32]
    L.wc_host_plan.restype = i32
    L.wc_host_plan.argtypes = [vp, u32, u64, u64, ctypes.POINTER(u32), vp, ctypes.POINTER(u32)]
    L.wc_encode_host.restype = i32
    L.wc_encode_host.argtypes = [ctypes.POINTER(HostEncodeItem), u32, vp, u64, u64, vp, vp, vp]
    L.wc_decode_host.restype = i32
    L.wc_decode_host.argtypes = [ctypes.POINTER(HostDecodeItem), u32, vp, u64, u64, vp, vp, vp,
                                 ctypes.POINTER(i32)]
    L.wc_chunk_ranges.restype = i32
    L.wc_chunk_ranges.argtypes = [vp, u64, u64, ctypes.POINTER(u64), ctypes.POINTER(u32)]
    L.wc12_encode_bound.restype = u64
    L.wc12_encode_bound.argtypes = [u64]
    L.wc12_scratch_bytes.restype = u64
    L.wc12_scratch_bytes.argtypes = [u64]
    L.wc12_encode.restype = i32
    L.wc12_encode.argtypes = [vp, u64, vp, u64, vp, u64, vp, vp]
    L.wc12_decode.restype = i32
    L.wc12_decode.argtypes = [vp, u64, vp, u64, vp, vp]
    L.wc12_read_header.restype = i32
    L.wc12_read_header.argtypes = [vp, u64, ctypes.POINTER(u64), ctypes.POINTER(u64), ctypes.POINTER(u32)]
    L.wc12_linear.restype = i32
    L.wc12_linear.argtypes = [vp, u64, u32, u32, vp, u32, vp, vp, vp]
    L.wc12_encode_batch.restype = i32
    L.wc12_encode_batch.argtypes = [ctypes.POINTER(Split12EncodeItem), u32, vp]
    L.wc12_decode_batch.restype = i32
    L.wc12_decode_batch.argtypes = [ctypes.POINTER(Split12DecodeItem), u32, vp, vp]
    L.wc12_plan_bytes.restype = u64
    L.wc12_plan_bytes.argtypes = [u32, u32, u64]
    L.wc12_plan.restype = i32
    L.wc12_plan.argtypes = [vp, u64, u32, u32, u64, vp, u64, vp, vp]
    L.wc12_linear_planned.restype = i32
    L.wc12_linear_planned.argtypes = [vp, u64, vp, u64, u32, u32, vp, u32, vp, vp, vp]
    L.wc_crc32_blocks.restype = i32
    L.wc_crc32_blocks.argtypes = [vp, u64, u64, vp, vp]
    L.wc_check_coder_division.restype = i32
    L.wc_check_coder_division.argtypes = [i32, u32, u32, vp, vp]
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().wc_status_string(code).decode()


def last_error() -> str:
    return load().wc_last_error().decode()


def _check(code: int, what: str):
    if code != OK:
        raise WCError(code, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def dtype_code(dtype: torch.dtype) -> int:
    try:
        return _DT[dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {dtype}: bf16, fp16, fp32, fp8 e4m3 and fp8 e5m2 only") from None


def encode_bound(n: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(load().wc_encode_bound(n, code))


def scratch_bytes(n: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(load().wc_scratch_bytes(n, code))


def read_header(cont) -> tuple[int, int, int]:
    """(n, dtype code, chunks) from a host copy of a container (bytes, numpy
    array or CPU uint8 tensor)."""
    if isinstance(cont, torch.Tensor):
        cont = cont.detach().cpu().numpy()
    import numpy as np
    buf = np.ascontiguousarray(np.frombuffer(bytes(cont), np.uint8) if isinstance(cont, (bytes, bytearray)) else cont,
                               dtype=np.uint8)
    n, dt, nc = ctypes.c_uint64(), ctypes.c_int32(), ctypes.c_uint64()
    _check(load().wc_read_header(buf.ctypes.data, buf.size, ctypes.byref(n), ctypes.byref(dt),
                                 ctypes.byref(nc)), "wc_read_header")
    return n.value, dt.value, nc.value


def _flat(t: torch.Tensor) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.reshape(-1)


def _align_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


class BatchEncoder:
    """Encodes a fixed list of tensor shapes/dtypes into preallocated device
    buffers with one wc_encode_batch call.  Containers stay on the device;
    `sizes` (u64 per tensor) is filled on the device."""

    def __init__(self, numels, dtypes, device="cuda"):
        self.numels = [int(n) for n in numels]
        self.codes = [d if isinstance(d, int) else dtype_code(d) for d in dtypes]
        self.device = torch.device(device)
        caps = [encode_bound(n, c) for n, c in zip(self.numels, self.codes)]
        scr = [scratch_bytes(n, c) for n, c in zip(self.numels, self.codes)]
        self.out_offsets, off = [], 0
        for c in caps:
            self.out_offsets.append(off)
            off = _align_up(off + c, 256)
        self.caps = caps
        self.out = torch.empty(max(off, 256), dtype=torch.uint8, device=self.device)
        self.scr_offsets, off = [], 0
        for c in scr:
            self.scr_offsets.append(off)
            off = _align_up(off + c, 256)
        self.scratch = torch.empty(max(off, 256), dtype=torch.uint8, device=self.device)
        self.sizes = torch.zeros(len(caps), dtype=torch.int64, device=self.device)
        self._items = (EncodeItem * len(caps))()
        self._key = None

    def containers(self, sizes=None) -> list[torch.Tensor]:
        """Views of the containers trimmed to size (reads the sizes back)."""
        if sizes is None:
            sizes = self.sizes.cpu().tolist()
        return [self.out[o:o + int(s)] for o, s in zip(self.out_offsets, sizes)]

    def prepare(self, tensors):
        """Bind input tensors once; run() then encodes them without any
        per-call Python work beyond one library call."""
        self._bind([_flat(t) for t in tensors])
        self._bound = list(tensors)
        return self

    def run(self, stream=None):
        _check(load().wc_encode_batch(self._items, len(self.numels), _stream(stream)),
               "wc_encode_batch")
        return self

    def encode(self, tensors, stream=None):
        self._bind([_flat(t) for t in tensors])
        return self.run(stream)

    def _bind(self, flats):
        if len(flats) != len(self.numels):
            raise ValueError("tensor count does not match the encoder")
        key = tuple(t.data_ptr() for t in flats)
        if key != self._key:
            base_o, base_s, base_z = self.out.data_ptr(), self.scratch.data_ptr(), self.sizes.data_ptr()
            for i, t in enumerate(flats):
                if t.numel() != self.numels[i] or dtype_code(t.dtype) != self.codes[i]:
                    raise ValueError(f"tensor {i} does not match the encoder's shape/dtype")
                it = self._items[i]
                it.in_ = t.data_ptr() if t.numel() else None
                it.n = t.numel()
                it.dtype = self.codes[i]
                it.reserved = 0
                it.out = base_o + self.out_offsets[i]
                it.out_cap = self.caps[i]
                it.scratch = base_s + self.scr_offsets[i]
                it.scratch_cap = scratch_bytes(self.numels[i], self.codes[i])
                it.out_size = base_z + 8 * i
            self._key = key


class BatchDecoder:
    """Decodes a fixed list of containers (device uint8 buffers) into
    preallocated outputs with one wc_decode_batch call."""

    def __init__(self, device="cuda"):
        self.device = torch.device(device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._items = None
        self._key = None

    def prepare(self, conts, outs, cont_bytes=None):
        self._bind(conts, outs, cont_bytes)
        self._n = len(conts)
        return self

    def run(self, stream=None):
        _check(load().wc_decode_batch(self._items, self._n, self.status.data_ptr(),
                                      _stream(stream)), "wc_decode_batch")
        return self

    def decode(self, conts, outs, cont_bytes=None, stream=None):
        self._bind(conts, outs, cont_bytes)
        self._n = len(conts)
        return self.run(stream)

    def _bind(self, conts, outs, cont_bytes):
        if cont_bytes is None:
            cont_bytes = [c.numel() for c in conts]
        key = tuple(c.data_ptr() for c in conts) + tuple(o.data_ptr() for o in outs) + tuple(cont_bytes)
        if key != self._key:
            self._items = (DecodeItem * len(conts))()
            for i, (c, o, nb) in enumerate(zip(conts, outs, cont_bytes)):
                of = _flat(o)
                it = self._items[i]
                it.cont = c.data_ptr()
                it.cont_bytes = int(nb)
                it.out = of.data_ptr() if of.numel() else None
                it.out_cap = of.numel() * of.element_size()
            self._key = key

    def check(self):
        """Synchronising read of the device status; raises on a bad container."""
        st = int(self.status.item())
        if st != OK:
            raise WCError(st, "decode (device status)")


# ---------------------------------------------------------------------------
# Convenience single-tensor calls (allocate through torch, sync to trim).
# ---------------------------------------------------------------------------
def encode(t: torch.Tensor, stream=None) -> torch.Tensor:
    """Container (device uint8 tensor, trimmed) for a bf16 / fp32 tensor."""
    f = _flat(t)
    code = dtype_code(f.dtype)
    n = f.numel()
    cap = encode_bound(n, code)
    out = torch.empty(cap, dtype=torch.uint8, device=f.device)
    scr = torch.empty(max(scratch_bytes(n, code), 256), dtype=torch.uint8, device=f.device)
    size = torch.zeros(1, dtype=torch.int64, device=f.device)
    _check(load().wc_encode(f.data_ptr() if n else None, n, code, out.data_ptr(), cap,
                            scr.data_ptr(), scr.numel(), size.data_ptr(), _stream(stream)),
           "wc_encode")
    return out[: int(size.item())]


def encode_noalloc(t: torch.Tensor, out: torch.Tensor, size: torch.Tensor, stream=None) -> None:
    """wc_encode_noalloc: encode into a caller-provided container buffer
    (`out`, uint8, >= encode_bound bytes) and size word (`size`, one int64),
    with the library-held scratch instead of a scratch buffer.  For callers
    that cannot allocate device memory at the call site; at most 16,252,928
    values.  Nothing is allocated and nothing is synchronised."""
    f = _flat(t)
    code = dtype_code(f.dtype)
    n = f.numel()
    _check(load().wc_encode_noalloc(f.data_ptr() if n else None, n, code, out.data_ptr(),
                                    out.numel(), size.data_ptr(), _stream(stream)),
           "wc_encode_noalloc")


def encode_batch(tensors, stream=None) -> list[torch.Tensor]:
    if not tensors:
        return []
    enc = BatchEncoder([t.numel() for t in tensors], [t.dtype for t in tensors],
                       device=tensors[0].device)
    enc.encode(tensors, stream)
    return [c.clone() for c in enc.containers()]


def decode(cont: torch.Tensor, shape=None, dtype=None, out=None, stream=None) -> torch.Tensor:
    """Decode a device container.  Without shape/dtype/out the header is
    copied to the host once to size the output."""
    if out is None:
        if shape is None or dtype is None:
            n, code, _ = read_header(cont[:64].cpu())
            dtype = _TORCH_DT[code]
            shape = (n,) if shape is None else shape
        out = torch.empty(shape, dtype=dtype, device=cont.device)
    of = _flat(out)
    status = torch.zeros(1, dtype=torch.int32, device=cont.device)
    _check(load().wc_decode(cont.data_ptr(), cont.numel(), of.data_ptr() if of.numel() else None,
                            of.numel() * of.element_size(), status.data_ptr(), _stream(stream)),
           "wc_decode")
    st = int(status.item())
    if st != OK:
        raise WCError(st, "wc_decode (device status)")
    return out


def decode_chunk(cont: torch.Tensor, k: int, dtype=None, stream=None) -> torch.Tensor:
    """Values [65536 k, min(n, 65536 (k + 1))) of a device container."""
    n, code, nc = read_header(cont[:64].cpu())
    if dtype is not None and dtype_code(dtype) != code:
        raise TypeError("dtype does not match the container")
    nvals = max(0, min(CHUNK, n - k * CHUNK)) if k < nc else 0
    out = torch.empty(max(nvals, 1), dtype=_TORCH_DT[code], device=cont.device)
    status = torch.zeros(1, dtype=torch.int32, device=cont.device)
    _check(load().wc_decode_chunk(cont.data_ptr(), cont.numel(), k, out.data_ptr(),
                                  nvals * _ELEM[code], status.data_ptr(), _stream(stream)),
           "wc_decode_chunk")
    st = int(status.item())
    if st != OK:
        raise WCError(st, "wc_decode_chunk (device status)")
    return out[:nvals]


def decode_batch(conts, shapes, dtypes, stream=None) -> list[torch.Tensor]:
    outs = [torch.empty(s, dtype=d, device=c.device) for c, s, d in zip(conts, shapes, dtypes)]
    dec = BatchDecoder(device=conts[0].device if conts else "cuda")
    dec.decode(conts, outs, stream=stream)
    dec.check()
    return outs


def chunk_ranges(prefix, k: int) -> list[tuple[int, int]]:
    """(offset, bytes) ranges of a container that decoding chunk k reads
    (wc_chunk_ranges); `prefix` is a host copy of the container's start
    (bytes or uint8 array) reaching at least the raw-plane offset."""
    import numpy as np
    buf = np.ascontiguousarray(np.frombuffer(prefix, np.uint8) if isinstance(prefix, (bytes, bytearray))
                               else prefix, dtype=np.uint8)
    out = (ctypes.c_uint64 * 8)()
    cnt = ctypes.c_uint32(0)
    _check(load().wc_chunk_ranges(buf.ctypes.data, buf.size, k, out, ctypes.byref(cnt)),
           "wc_chunk_ranges")
    return [(int(out[2 * i]), int(out[2 * i + 1])) for i in range(cnt.value)]


# ---------------------------------------------------------------------------
# Split12 serving format (include/wc_split12.h): bf16 only.

def split12_encode_bound(n: int) -> int:
    return int(load().wc12_encode_bound(n))


def split12_scratch_bytes(n: int) -> int:
    return int(load().wc12_scratch_bytes(n))


def split12_read_header(cont, cont_bytes: int | None = None) -> tuple[int, int, int]:
    """(n, exceptions, codebook entries) of a Split12 container, from a host
    copy of (at least) its first 64 bytes (bytes or uint8 array); cont_bytes
    is the container's size (default: the copy's)."""
    import numpy as np
    buf = np.ascontiguousarray(np.frombuffer(cont, np.uint8) if isinstance(cont, (bytes, bytearray))
                               else cont, dtype=np.uint8)
    size = buf.size if cont_bytes is None else int(cont_bytes)
    if buf.size < 64:
        raise WCError(ERR_CORRUPT, "wc12_read_header")
    n, ne, k = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint32()
    _check(load().wc12_read_header(buf.ctypes.data, size, ctypes.byref(n), ctypes.byref(ne),
                                   ctypes.byref(k)), "wc12_read_header")
    return n.value, ne.value, k.value


def split12_encode(t: torch.Tensor, stream=None) -> torch.Tensor:
    """Split12 container (device uint8, trimmed) of a bf16 CUDA tensor."""
    if t.dtype != torch.bfloat16:
        raise TypeError("Split12 takes bf16 tensors")
    f = _flat(t)
    n = f.numel()
    out = torch.empty(split12_encode_bound(n), dtype=torch.uint8, device=f.device)
    scr = torch.empty(split12_scratch_bytes(n), dtype=torch.uint8, device=f.device)
    size = torch.zeros(1, dtype=torch.int64, device=f.device)
    _check(load().wc12_encode(f.data_ptr() if n else None, n, out.data_ptr(), out.numel(),
                              scr.data_ptr(), scr.numel(), size.data_ptr(), _stream(stream)),
           "wc12_encode")
    return out[: int(size.item())]


def split12_decode(cont: torch.Tensor, shape=None, out=None, stream=None) -> torch.Tensor:
    """Decode a device Split12 container into bf16 (shape from the header's
    value count, bytes 8..15, unless given)."""
    if out is None:
        if shape is None:
            shape = (int(cont[8:16].cpu().numpy().view("<u8")[0]),)
        out = torch.empty(shape, dtype=torch.bfloat16, device=cont.device)
    of = _flat(out)
    status = torch.zeros(1, dtype=torch.int32, device=cont.device)
    _check(load().wc12_decode(cont.data_ptr(), cont.numel(), of.data_ptr() if of.numel() else None,
                              of.numel() * 2, status.data_ptr(), _stream(stream)), "wc12_decode")
    st = int(status.item())
    if st != OK:
        raise WCError(st, "wc12_decode (device status)")
    return out


def split12_encode_batch(tensors, stream=None) -> list[torch.Tensor]:
    """Split12 containers of many bf16 CUDA tensors, one launch per encoder
    kernel for the whole list (wc12_encode_batch)."""
    flats = []
    for t in tensors:
        if t.dtype != torch.bfloat16:
            raise TypeError("Split12 takes bf16 tensors")
        flats.append(_flat(t))
    outs, scrs, sizes = [], [], []
    items = (Split12EncodeItem * max(1, len(flats)))()
    for i, f in enumerate(flats):
        n = f.numel()
        outs.append(torch.empty(split12_encode_bound(n), dtype=torch.uint8, device=f.device))
        scrs.append(torch.empty(split12_scratch_bytes(n), dtype=torch.uint8, device=f.device))
        sizes.append(torch.zeros(1, dtype=torch.int64, device=f.device))
        items[i] = Split12EncodeItem(f.data_ptr() if n else None, n, outs[-1].data_ptr(), outs[-1].numel(),
                                     scrs[-1].data_ptr(), scrs[-1].numel(), sizes[-1].data_ptr())
    if flats:
        _check(load().wc12_encode_batch(items, len(flats), _stream(stream)), "wc12_encode_batch")
    return [o[: int(z.item())] for o, z in zip(outs, sizes)]


def split12_decode_batch(conts, shapes, stream=None) -> list[torch.Tensor]:
    """Decode many device Split12 containers into bf16 tensors of the given
    shapes, one launch (wc12_decode_batch)."""
    if len(conts) != len(shapes):
        raise ValueError("one shape per container")
    outs = []
    items = (Split12DecodeItem * max(1, len(conts)))()
    dev = conts[0].device if conts else None
    for i, (c, sh) in enumerate(zip(conts, shapes)):
        o = torch.empty(sh, dtype=torch.bfloat16, device=c.device)
        outs.append(o)
        items[i] = Split12DecodeItem(c.data_ptr(), c.numel(), o.data_ptr() if o.numel() else None, o.numel())
    if conts:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        _check(load().wc12_decode_batch(items, len(conts), status.data_ptr(), _stream(stream)),
               "wc12_decode_batch")
        st = int(status.item())
        if st != OK:
            raise WCError(st, "wc12_decode_batch (device status)")
    return outs


def split12_plan_bytes(N: int, K: int, ne: int) -> int:
    return int(load().wc12_plan_bytes(N, K, ne))


def split12_plan(cont: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    """The serving plan of a Split12 container on the device (wc12_plan): its
    exceptions grouped by the linear layer's 128 x 64 tiles.  Reads the
    container's header to the host once, for its exception count."""
    _n, ne, _k = split12_read_header(cont[:64].cpu().numpy(), cont.numel())
    plan = torch.empty(split12_plan_bytes(N, K, ne), dtype=torch.uint8, device=cont.device)
    status = torch.zeros(1, dtype=torch.int32, device=cont.device)
    _check(load().wc12_plan(cont.data_ptr(), cont.numel(), N, K, ne, plan.data_ptr(), plan.numel(),
                            status.data_ptr(), _stream(stream)), "wc12_plan")
    st = int(status.item())
    if st != OK:
        raise WCError(st, "wc12_plan (device status)")
    return plan


def split12_linear(cont: torch.Tensor, N: int, K: int, x: torch.Tensor, plan=None,
                   stream=None) -> torch.Tensor:
    """Y = x W^T (fp32, M x N) with W (N x K bf16) given as a Split12
    container on the device (wc12_linear, or wc12_linear_planned with the
    container's plan)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != K:
        raise ValueError("x must be a 2-D bf16 tensor with K columns")
    xf = x.contiguous()
    y = torch.empty(x.shape[0], N, dtype=torch.float32, device=x.device)
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    if plan is None:
        _check(load().wc12_linear(cont.data_ptr(), cont.numel(), N, K, xf.data_ptr(), x.shape[0],
                                  y.data_ptr(), status.data_ptr(), _stream(stream)), "wc12_linear")
    else:
        _check(load().wc12_linear_planned(cont.data_ptr(), cont.numel(), plan.data_ptr(), plan.numel(), N, K,
                                          xf.data_ptr(), x.shape[0], y.data_ptr(), status.data_ptr(),
                                          _stream(stream)), "wc12_linear_planned")
    st = int(status.item())
    if st != OK:
        raise WCError(st, "wc12_linear (device status)")
    return y


def check_coder_division(wide: bool, f_first: int, f_last: int, stream=None) -> tuple[int, int]:
    """wc_check_coder_division: (mismatches, one failing f << 32 | x) of the
    encoder's division by f over every state x < f 2^20 (synchronises)."""
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    _check(load().wc_check_coder_division(1 if wide else 0, f_first, f_last, res.data_ptr(),
                                          _stream(stream)), "wc_check_coder_division")
    out = res.cpu().tolist()
    return int(out[0]), int(out[1])


CRC_BLOCK = 1 << 20


def crc32_blocks(buf: torch.Tensor, block_bytes: int = CRC_BLOCK, stream=None) -> torch.Tensor:
    """CRC-32 (zlib's code) of each block_bytes-sized block of a contiguous
    device tensor's bytes (wc_crc32_blocks); int32 tensor on the device, one
    entry per block, the bits of the unsigned CRC."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buffer must be a contiguous CUDA tensor")
    nbytes = buf.numel() * buf.element_size()
    nb = -(-nbytes // block_bytes) if block_bytes > 0 else 0
    out = torch.empty(max(nb, 1), dtype=torch.int32, device=buf.device)
    _check(load().wc_crc32_blocks(buf.data_ptr() if nbytes else None, nbytes, block_bytes,
                                  out.data_ptr(), _stream(stream)), "wc_crc32_blocks")
    return out[:nb]


# ---------------------------------------------------------------------------
# Host-resident tensors through the device in windows (wc_encode_host /
# wc_decode_host): the library runs the copy / kernel pipeline; this class
# only owns the device workspace, the three streams and pinned host buffers.

def host_plan(footprints, slot_area: int, window_bytes: int = 0) -> tuple[int, list[int]]:
    """(slots, window ends) of wc_host_plan for the given item footprints."""
    import numpy as np
    fp = np.ascontiguousarray(np.asarray(footprints, dtype=np.uint64))
    ends = np.zeros(max(1, fp.size), np.uint32)
    k, w = ctypes.c_uint32(), ctypes.c_uint32()
    _check(load().wc_host_plan(fp.ctypes.data if fp.size else None, fp.size, slot_area,
                               window_bytes, ctypes.byref(k), ends.ctypes.data, ctypes.byref(w)),
           "wc_host_plan")
    return k.value, ends[:w.value].tolist()


def host_encode_footprint(n: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(load().wc_host_encode_footprint(n, code))


def host_decode_footprint(cont_bytes: int, n: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(load().wc_host_decode_footprint(cont_bytes, n, code))


def _host_flat(t: torch.Tensor) -> torch.Tensor:
    if t.is_cuda:
        raise ValueError("host pipeline: tensor must be in host memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.reshape(-1)


class HostCodec:
    """Encodes host tensors into host containers and decodes them back,
    streaming windows of about `window_bytes` of slot space through a device
    workspace of `work_bytes` with three CUDA streams (copy in, kernels, copy
    out).  Host buffers should be pinned (`torch.empty(..., pin_memory=True)`)
    for the copies to overlap."""

    def __init__(self, work_bytes: int, device="cuda", window_bytes: int = 128 << 20):
        self.device = torch.device(device)
        self.window_bytes = int(window_bytes)
        self.work = torch.empty(int(work_bytes), dtype=torch.uint8, device=self.device)
        self.streams = [torch.cuda.Stream(device=self.device) for _ in range(3)]

    def _s(self):
        return [s.cuda_stream for s in self.streams]

    def encode_buffers(self, tensors, pin=True) -> tuple[list[torch.Tensor], torch.Tensor]:
        """Host buffers of wc_encode_bound bytes for the given tensors, and the
        host u64 size array; reuse them across encode() calls."""
        outs = [torch.empty(max(16, encode_bound(t.numel(), t.dtype)), dtype=torch.uint8,
                            pin_memory=pin) for t in tensors]
        return outs, torch.zeros(len(tensors), dtype=torch.int64)

    def encode(self, tensors, outs=None, sizes=None) -> list[torch.Tensor]:
        """Containers (host uint8 views, trimmed) of host tensors."""
        flats = [_host_flat(t) for t in tensors]
        if outs is None or sizes is None:
            outs, sizes = self.encode_buffers(tensors, pin=all(t.is_pinned() for t in flats))
        items = (HostEncodeItem * len(flats))()
        for i, t in enumerate(flats):
            it = items[i]
            it.h_in = t.data_ptr() if t.numel() else None
            it.n = t.numel()
            it.dtype = dtype_code(t.dtype)
            it.reserved = 0
            it.h_out = outs[i].data_ptr()
            it.h_out_cap = outs[i].numel()
            it.h_out_size = sizes.data_ptr() + 8 * i
        si, sc, so = self._s()
        _check(load().wc_encode_host(items, len(flats), self.work.data_ptr(), self.work.numel(),
                                     self.window_bytes, si, sc, so), "wc_encode_host")
        return [o[:int(z)] for o, z in zip(outs, sizes.tolist())]

    def decode(self, conts, outs=None, pin=True) -> list[torch.Tensor]:
        """Decoded host tensors (1-D) of host containers."""
        hdr = [read_header(c) for c in conts]
        if outs is None:
            outs = [torch.empty(n, dtype=_TORCH_DT[dt], pin_memory=pin) for n, dt, _ in hdr]
        items = (HostDecodeItem * len(conts))()
        for i, (c, o) in enumerate(zip(conts, outs)):
            if c.is_cuda or not c.is_contiguous():
                raise ValueError("host pipeline: containers must be contiguous host buffers")
            it = items[i]
            it.h_cont = c.data_ptr()
            it.cont_bytes = c.numel()
            it.h_out = o.data_ptr() if o.numel() else None
            it.out_cap = o.numel() * o.element_size()
        st = ctypes.c_int32()
        si, sc, so = self._s()
        _check(load().wc_decode_host(items, len(conts), self.work.data_ptr(), self.work.numel(),
                                     self.window_bytes, si, sc, so, ctypes.byref(st)),
               "wc_decode_host")
        _check(st.value, "wc_decode_host (device status)")
        return outs
