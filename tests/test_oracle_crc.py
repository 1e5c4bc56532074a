"""Pins of the oracle's CRC-32 ("seedpack 0.2.0 -> 0.2.2", README: a CRC32
per archive chunk), fixed by things other than the oracle itself: the
catalogue check value, the residue that a message followed by its own CRC
leaves, and zlib's implementation of the same code."""
import struct
import zlib

import numpy as np
import pytest


def test_check_values(orc):
    # the CRC catalogue's check value for CRC-32 (ISO-HDLC / zlib)
    assert orc.crc32(b"123456789") == 0xCBF43926
    assert orc.crc32(b"") == 0
    assert orc.crc32(b"a") == 0xE8B7BE43
    assert orc.crc32(b"\0" * 4) == 0x2144DF1C


def test_residue_of_message_and_its_crc(orc):
    # appending a message's CRC (little-endian) leaves a fixed residue
    rng = np.random.default_rng(3)
    for n in (0, 1, 7, 100, 4096):
        m = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        c = orc.crc32(m)
        assert orc.crc32(m + struct.pack("<I", c)) == 0x2144DF1C


@pytest.mark.parametrize("n", [1, 2, 3, 4, 15, 16, 17, 255, 4095, 4096, 4097, 65537, 1 << 20])
def test_matches_zlib(orc, n):
    data = np.random.default_rng(n).integers(0, 256, n, dtype=np.uint8)
    assert orc.crc32(data) == zlib.crc32(data.tobytes())


def test_blocks(orc):
    data = np.random.default_rng(8).integers(0, 256, 3 * 8192 + 5, dtype=np.uint8)
    got = orc.crc32_blocks(data, 8192)
    assert got.size == 4
    for i in range(4):
        assert got[i] == zlib.crc32(data[i * 8192:(i + 1) * 8192].tobytes())
    assert orc.crc32_blocks(data[:0], 8192).size == 0
    assert np.array_equal(orc.crc32_blocks(data[:8192], 8192), [zlib.crc32(data[:8192].tobytes())])
