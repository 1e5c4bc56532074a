"""A file of named containers with an index: whole weight sets saved in one
file and read back by name, whole or one chunk at a time ("PTWM", Random
access: a tensor index over the compressed file; "seedpack 0.2.0 -> 0.2.2",
README: a container of many tensors plus an index).

Layout (little-endian):
    0   "WCA1"
    4   u32 version (1)
    8   u32 number of entries
    12  u32 checksum block B in bytes (0: no checksums)
    16  u64 offset of the index
    24  u64 bytes of the index
    32  the containers, each starting on a 16-byte boundary, zero padding
    index: per entry  u16 name bytes, the UTF-8 name, u8 dtype code,
           u8 number of dimensions, u64 per dimension, u64 container offset,
           u64 container bytes, then (B > 0) one u32 CRC-32 per B-byte block
           of the container, the last block short

The containers are exactly those of the library: the rANS storage format
(include/wc.h, magic "WCZ1") or the Split12 serving format
(include/wc_split12.h, magic "W12C", bf16 only), told apart by their magic;
this module only places them in a file and finds them again.  Encoding, decoding and the
checksums ("seedpack 0.2.0 -> 0.2.2", README: a CRC32 per archive chunk) run
on the GPU through the binding.
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


def _nblocks(nbytes: int, block: int) -> int:
    return -(-nbytes // block) if block else 0


def write(path: str, entries, crc_block: int = 0) -> None:
    """Write an archive from (name, dtype code, shape, container bytes[,
    CRCs]) entries, in the given order.  With crc_block > 0 every entry
    carries the CRC-32 of each crc_block-byte block of its container."""
    entries = [tuple(e) for e in entries]
    names = [e[0] for e in entries]
    if len(set(names)) != len(names):
        raise ValueError("duplicate tensor names")
    if crc_block < 0 or crc_block >= 1 << 32:
        raise ValueError("checksum block size out of range")
    offsets, off = [], _HEAD.size
    for e in entries:
        offsets.append(off)
        off = _align16(off + len(e[3]))
    index = bytearray()
    for e, o in zip(entries, offsets):
        name, code, shape, cont = e[:4]
        nb = name.encode("utf-8")
        if len(nb) > 0xFFFF or len(shape) > 255:
            raise ValueError(f"entry {name!r}: name or rank too large")
        index += struct.pack("<H", len(nb)) + nb + struct.pack("<BB", int(code), len(shape))
        index += struct.pack(f"<{len(shape)}Q", *[int(d) for d in shape])
        index += struct.pack("<QQ", o, len(cont))
        crcs = np.asarray(e[4] if len(e) > 4 and e[4] is not None else [], dtype=np.uint32)
        if crcs.size != _nblocks(len(cont), crc_block):
            raise ValueError(f"entry {name!r}: {crcs.size} checksums for "
                             f"{_nblocks(len(cont), crc_block)} blocks")
        index += crcs.astype("<u4").tobytes()
    with open(path, "wb") as fh:
        fh.write(_HEAD.pack(MAGIC, VERSION, len(entries), crc_block, off, len(index)))
        pos = _HEAD.size
        for e, o in zip(entries, offsets):
            fh.write(b"\0" * (o - pos))
            fh.write(bytes(e[3]))
            pos = o + len(e[3])
        fh.write(b"\0" * (off - pos))
        fh.write(index)


def save(path: str, tensors: dict, stream=None, crc_block: int = wc.CRC_BLOCK,
         codec: str = "rans") -> None:
    """Encode every tensor (CUDA tensors) and write the containers to an
    archive under their names, each checksummed on the device (crc_block 0:
    none).  codec "rans": the storage format, one batched launch per kernel;
    "split12": the serving format (bf16 tensors only), which wc12_linear
    multiplies without decoding."""
    items = list(tensors.items())
    if codec == "rans":
        conts = wc.encode_batch([t.contiguous() for _, t in items], stream)
    elif codec == "split12":
        conts = [wc.split12_encode(t.contiguous(), stream) for _, t in items]
    else:
        raise ValueError(f"unknown codec {codec!r}")
    crcs = [wc.crc32_blocks(c, crc_block, stream) if crc_block else None for c in conts]
    write(path, [(name, wc.dtype_code(t.dtype), tuple(t.shape), c.cpu().numpy().tobytes(),
                  None if k is None else k.cpu().numpy().view(np.uint32))
                 for (name, t), c, k in zip(items, conts, crcs)], crc_block)


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
        magic, version, count, crc_block, ioff, ibytes = _HEAD.unpack_from(self._mm, 0)
        if magic != MAGIC or version != VERSION or ioff + ibytes > size:
            raise ValueError("not an archive or unsupported version")
        self.crc_block = crc_block
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
            if off < _HEAD.size or off + nbytes > ioff or off % 16:
                raise ValueError(f"entry {name!r}: container outside the data section")
            nck = _nblocks(nbytes, crc_block)
            if p + 4 * nck > ioff + ibytes:
                raise ValueError("index runs past its stated size")
            crcs = np.frombuffer(self._mm, dtype="<u4", count=nck, offset=p).astype(np.uint32)
            p += 4 * nck
            if code not in wc._TORCH_DT:
                raise ValueError(f"entry {name!r}: unknown dtype code {code}")
            if name in self._entries:
                raise ValueError(f"entry {name!r} appears twice")
            head = bytes(self._mm[off:off + min(nbytes, 64)])
            if head[:4] == b"W12C":
                codec = "split12"
                n, _, _ = wc.split12_read_header(head, nbytes)
                hcode = wc.BF16
            else:
                codec = "rans"
                n, hcode, _ = wc.read_header(head)
            if hcode != code or n != int(np.prod(shape, dtype=np.uint64)):
                raise ValueError(f"entry {name!r}: container header disagrees with the index")
            self._entries[name] = (code, tuple(shape), off, nbytes, crcs, codec)
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
        code, shape, _, nbytes = self._entries[name][:4]
        return wc._TORCH_DT[code], shape, nbytes

    def codec(self, name: str) -> str:
        """"rans" (storage format) or "split12" (serving format)."""
        return self._entries[name][5]

    def checksums(self, name: str) -> np.ndarray:
        """The stored CRC-32 of each checksum block of the entry's container
        (empty when the archive has none)."""
        return self._entries[name][4].copy()

    def container(self, name: str) -> np.ndarray:
        """A copy of the entry's container bytes."""
        _, _, off, nbytes = self._entries[name][:4]
        return np.frombuffer(self._mm, dtype=np.uint8, count=nbytes, offset=off).copy()

    def device_container(self, name: str, device="cuda", stream=None, verify: bool = True) -> torch.Tensor:
        """The entry's container on the device (checksums checked unless
        verify is False): the operand wc.split12_linear takes for a Split12
        entry."""
        return self._device_container(name, device, verify, stream)

    def _device_container(self, name: str, device, verify: bool, stream) -> torch.Tensor:
        cont = torch.from_numpy(self.container(name)).to(device)
        if verify and self.crc_block:
            bad = self._bad_blocks(name, cont, stream)
            if bad:
                raise ValueError(f"entry {name!r}: checksum mismatch in block(s) {bad[:8]}")
        return cont

    def _bad_blocks(self, name: str, cont: torch.Tensor, stream) -> list[int]:
        got = wc.crc32_blocks(cont, self.crc_block, stream).cpu().numpy().view(np.uint32)
        return np.nonzero(got != self._entries[name][4])[0].tolist()

    def verify(self, name: str, device="cuda", stream=None) -> list[int]:
        """Indices of the checksum blocks of an entry whose CRC-32, computed on
        the device, differs from the stored one (empty: intact, or no
        checksums in this archive)."""
        if not self.crc_block:
            return []
        cont = torch.from_numpy(self.container(name)).to(device)
        return self._bad_blocks(name, cont, stream)

    def load(self, name: str, device="cuda", stream=None, verify: bool = True) -> torch.Tensor:
        """Decode one tensor onto the device (checksums checked first unless
        verify is False; a mismatch raises ValueError)."""
        code, shape = self._entries[name][:2]
        cont = self._device_container(name, device, verify, stream)
        if self.codec(name) == "split12":
            return wc.split12_decode(cont, shape=shape, stream=stream)
        return wc.decode(cont, shape=shape, dtype=wc._TORCH_DT[code], stream=stream)

    def load_chunk(self, name: str, k: int, device="cuda", stream=None,
                   verify: bool = True) -> torch.Tensor:
        """Values k * 65536 .. of one tensor (1-D), decoding that chunk only.
        Only the bytes the chunk needs leave the file: the header and tables,
        the chunk's raw-plane bytes and its payload (wc_chunk_ranges), widened
        to whole checksum blocks when those are checked."""
        code, _, off, nbytes, crcs, codec = self._entries[name]
        if codec != "rans":
            raise ValueError(f"entry {name!r}: chunk access needs the rANS storage format")
        (off_raw,) = struct.unpack_from("<Q", self._mm, off + 32)
        if off_raw > nbytes:
            raise ValueError(f"entry {name!r}: container header out of range")
        ranges = wc.chunk_ranges(bytes(self._mm[off:off + off_raw]), k)
        check = verify and self.crc_block > 0
        if check:
            B = self.crc_block
            blocks = sorted({b for o, n in ranges if n for b in range(o // B, (o + n - 1) // B + 1)})
            ranges = [(b * B, min(B, nbytes - b * B)) for b in blocks]
        cont = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        for o, n in ranges:
            if o + n > nbytes:
                raise ValueError(f"entry {name!r}: chunk {k} reaches past its container")
            cont[o:o + n].copy_(torch.from_numpy(
                np.frombuffer(self._mm, dtype=np.uint8, count=n, offset=off + o).copy()))
        if check:
            got = wc.crc32_blocks(cont, self.crc_block, stream).cpu().numpy().view(np.uint32)
            bad = [b for b in blocks if got[b] != crcs[b]]
            if bad:
                raise ValueError(f"entry {name!r}: checksum mismatch in block(s) {bad[:8]}")
        return wc.decode_chunk(cont, k, dtype=wc._TORCH_DT[code], stream=stream)

    def load_all(self, names=None, device="cuda", stream=None, verify: bool = True) -> dict:
        """Decode several tensors: the rANS entries with one batched launch,
        Split12 entries one call each."""
        names = self.names() if names is None else list(names)
        rans = [n for n in names if self.codec(n) == "rans"]
        conts = [self._device_container(n, device, verify, stream) for n in rans]
        shapes = [self._entries[n][1] for n in rans]
        dtypes = [wc._TORCH_DT[self._entries[n][0]] for n in rans]
        got = dict(zip(rans, wc.decode_batch(conts, shapes, dtypes, stream)))
        for n in names:
            if n not in got:
                got[n] = self.load(n, device, stream, verify)
        return {n: got[n] for n in names}
