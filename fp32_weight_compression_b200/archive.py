"""A file of named containers with an index: whole weight sets saved in one
file and read back by name, whole or one chunk at a time ("PTWM", Random
access: a tensor index over the compressed file; "seedpack 0.2.0 -> 0.2.2",
README: a container of many tensors plus an index).

Layout (little-endian):
    0   "WCA1"
    4   u32 version (1)
    8   u32 number of entries
    12  u32 0
    16  u64 offset of the index
    24  u64 bytes of the index
    32  the containers, each starting on a 16-byte boundary, zero padding
    index: per entry  u16 name bytes, the UTF-8 name, u8 dtype code,
           u8 number of dimensions, u64 per dimension, u64 container offset,
           u64 container bytes

The containers are exactly those of the library (include/wc.h); this module
only places them in a file and finds them again.  Encoding and decoding run on
the GPU through the binding.
"""
from __future__ import annotations

import mmap
import os
import struct

import numpy as np
import torch

from . import wc

MAGIC = b"WCA1"
VERSION = 1
_HEAD = struct.Struct("<4sIII QQ")


def _align16(v: int) -> int:
    return (v + 15) // 16 * 16


def write(path: str, entries) -> None:
    """Write an archive from (name, dtype code, shape, container bytes)
    entries, in the given order."""
    entries = list(entries)
    names = [e[0] for e in entries]
    if len(set(names)) != len(names):
        raise ValueError("duplicate tensor names")
    offsets, off = [], _HEAD.size
    for _, _, _, cont in entries:
        offsets.append(off)
        off = _align16(off + len(cont))
    index = bytearray()
    for (name, code, shape, cont), o in zip(entries, offsets):
        nb = name.encode("utf-8")
        if len(nb) > 0xFFFF or len(shape) > 255:
            raise ValueError(f"entry {name!r}: name or rank too large")
        index += struct.pack("<H", len(nb)) + nb + struct.pack("<BB", int(code), len(shape))
        index += struct.pack(f"<{len(shape)}Q", *[int(d) for d in shape])
        index += struct.pack("<QQ", o, len(cont))
    with open(path, "wb") as fh:
        fh.write(_HEAD.pack(MAGIC, VERSION, len(entries), 0, off, len(index)))
        pos = _HEAD.size
        for (_, _, _, cont), o in zip(entries, offsets):
            fh.write(b"\0" * (o - pos))
            fh.write(bytes(cont))
            pos = o + len(cont)
        fh.write(b"\0" * (off - pos))
        fh.write(index)


def save(path: str, tensors: dict, stream=None) -> None:
    """Encode every tensor (CUDA tensors; one batched launch per kernel) and
    write them to an archive under their names."""
    items = list(tensors.items())
    conts = wc.encode_batch([t.contiguous() for _, t in items], stream)
    write(path, [(name, wc.dtype_code(t.dtype), tuple(t.shape), c.cpu().numpy().tobytes())
                 for (name, t), c in zip(items, conts)])


class Archive:
    """Read side: the index at open, containers on demand (memory-mapped)."""

    def __init__(self, path: str):
        self._fh = open(path, "rb")
        size = os.fstat(self._fh.fileno()).st_size
        if size < _HEAD.size:
            self._fh.close()
            raise ValueError("not an archive: too short")
        self._mm = mmap.mmap(self._fh.fileno(), 0, access=mmap.ACCESS_READ)
        try:
            self._read_index(size)
        except (struct.error, wc.WCError) as e:
            self.close()
            raise ValueError(f"damaged archive: {e}") from None
        except Exception:
            self.close()
            raise

    def _read_index(self, size: int) -> None:
        magic, version, count, _, ioff, ibytes = _HEAD.unpack_from(self._mm, 0)
        if magic != MAGIC or version != VERSION or ioff + ibytes > size:
            raise ValueError("not an archive or unsupported version")
        self._entries = {}
        p = ioff
        for _ in range(count):
            (nlen,) = struct.unpack_from("<H", self._mm, p)
            p += 2
            name = bytes(self._mm[p:p + nlen]).decode("utf-8")
            p += nlen
            code, ndim = struct.unpack_from("<BB", self._mm, p)
            p += 2
            shape = struct.unpack_from(f"<{ndim}Q", self._mm, p)
            p += 8 * ndim
            off, nbytes = struct.unpack_from("<QQ", self._mm, p)
            p += 16
            if p > ioff + ibytes:
                raise ValueError("index runs past its stated size")
            if off < _HEAD.size or off + nbytes > ioff or off % 16:
                raise ValueError(f"entry {name!r}: container outside the data section")
            if code not in wc._TORCH_DT:
                raise ValueError(f"entry {name!r}: unknown dtype code {code}")
            if name in self._entries:
                raise ValueError(f"entry {name!r} appears twice")
            n, hcode, _ = wc.read_header(bytes(self._mm[off:off + min(nbytes, 64)]))
            if hcode != code or n != int(np.prod(shape, dtype=np.uint64)):
                raise ValueError(f"entry {name!r}: container header disagrees with the index")
            self._entries[name] = (code, tuple(shape), off, nbytes)
        if p != ioff + ibytes:
            raise ValueError("index size does not match its entries")

    def close(self) -> None:
        self._mm.close()
        self._fh.close()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def names(self) -> list[str]:
        return list(self._entries)

    def __len__(self) -> int:
        return len(self._entries)

    def __contains__(self, name) -> bool:
        return name in self._entries

    def info(self, name: str) -> tuple[torch.dtype, tuple, int]:
        """(dtype, shape, container bytes) of an entry."""
        code, shape, _, nbytes = self._entries[name]
        return wc._TORCH_DT[code], shape, nbytes

    def container(self, name: str) -> np.ndarray:
        """A copy of the entry's container bytes."""
        _, _, off, nbytes = self._entries[name]
        return np.frombuffer(self._mm, dtype=np.uint8, count=nbytes, offset=off).copy()

    def _device_container(self, name: str, device) -> torch.Tensor:
        return torch.from_numpy(self.container(name)).to(device)

    def load(self, name: str, device="cuda", stream=None) -> torch.Tensor:
        """Decode one tensor onto the device."""
        code, shape, _, _ = self._entries[name]
        cont = self._device_container(name, device)
        return wc.decode(cont, shape=shape, dtype=wc._TORCH_DT[code], stream=stream)

    def load_chunk(self, name: str, k: int, device="cuda", stream=None) -> torch.Tensor:
        """Values k * 65536 .. of one tensor (1-D), decoding that chunk only."""
        code = self._entries[name][0]
        cont = self._device_container(name, device)
        return wc.decode_chunk(cont, k, dtype=wc._TORCH_DT[code], stream=stream)

    def load_all(self, names=None, device="cuda", stream=None) -> dict:
        """Decode several tensors with one batched launch."""
        names = self.names() if names is None else list(names)
        conts = [self._device_container(n, device) for n in names]
        shapes = [self._entries[n][1] for n in names]
        dtypes = [wc._TORCH_DT[self._entries[n][0]] for n in names]
        outs = wc.decode_batch(conts, shapes, dtypes, stream)
        return dict(zip(names, outs))
