"""The archive file (named containers plus an index) without a GPU: containers
written by the oracle come back byte for byte under their names, with their
dtypes and shapes, and damaged or inconsistent files are refused."""
import struct

import numpy as np
import pytest

import workloads

C = 65536


@pytest.fixture(scope="module")
def arc():
    from fp32_weight_compression_b200 import archive, build
    build.build()
    return archive


def _entries(orc):
    rng = np.random.default_rng(5)
    bf = workloads.rne_bf16(rng.standard_normal(2 * C + 7).astype(np.float32) * np.float32(0.02))
    f32 = (rng.standard_normal(C + 3).astype(np.float32) * np.float32(0.02)).view(np.uint32)
    f16 = (rng.standard_normal(999) * 0.05).astype(np.float16)
    f8 = ((rng.integers(0, 2, 4097) << 7) | (np.clip(rng.normal(6, 1.3, 4097), 0, 15).astype(np.int64) << 3)
          | rng.integers(0, 8, 4097)).astype(np.uint8)
    return [
        ("layers.0.mlp.weight", 1, (3, 43693), bf, orc.encode(bf)),
        ("emb/é", 2, (C + 3,), f32, orc.encode(f32)),
        ("h", 3, (27, 37), f16, orc.encode(f16)),
        ("fp8.w", 4, (4097,), f8, orc.encode(f8)),
        ("empty", 1, (0, 5), np.zeros(0, np.uint16), orc.encode(np.zeros(0, np.uint16))),
    ]


def test_write_and_read_back(orc, arc, tmp_path):
    import torch
    ents = _entries(orc)
    assert ents[0][2][0] * ents[0][2][1] == ents[0][3].size
    path = str(tmp_path / "w.wca")
    arc.write(path, [(n, c, s, cont.tobytes()) for n, c, s, _, cont in ents])
    want_dt = {1: torch.bfloat16, 2: torch.float32, 3: torch.float16, 4: torch.float8_e4m3fn}
    with arc.Archive(path) as a:
        assert a.names() == [e[0] for e in ents]
        assert len(a) == len(ents) and "h" in a and "nope" not in a
        for name, code, shape, bits, cont in ents:
            dt, sh, nbytes = a.info(name)
            assert dt == want_dt[code] and sh == shape and nbytes == cont.size
            got = a.container(name)
            assert np.array_equal(got, cont)
            # the stored container still decodes to the values (oracle decoder)
            assert np.array_equal(orc.decode(got).view(np.uint8), bits.view(np.uint8))
    # every container starts on a 16-byte boundary
    raw = open(path, "rb").read()
    ioff, ibytes = struct.unpack_from("<QQ", raw, 16)
    assert ioff + ibytes == len(raw)
    for _, _, _, _, cont in ents:
        pos = raw.find(cont.tobytes(), 32)
        assert pos >= 32 and pos % 16 == 0


def _one(orc):
    bits = workloads.rne_bf16(np.random.default_rng(9).standard_normal(C + 1).astype(np.float32))
    return bits, orc.encode(bits)


def test_duplicate_names_refused(orc, arc, tmp_path):
    _, cont = _one(orc)
    with pytest.raises(ValueError):
        arc.write(str(tmp_path / "d.wca"), [("a", 1, (C + 1,), cont.tobytes())] * 2)


def test_damaged_files_refused(orc, arc, tmp_path):
    _, cont = _one(orc)
    path = tmp_path / "g.wca"
    arc.write(str(path), [("a", 1, (C + 1,), cont.tobytes())])
    good = path.read_bytes()

    def reopen(data):
        p = tmp_path / "bad.wca"
        p.write_bytes(data)
        a = arc.Archive(str(p))
        a.close()

    reopen(good)  # intact
    with pytest.raises(ValueError):
        reopen(b"XXXX" + good[4:])                                # magic
    with pytest.raises(ValueError):
        reopen(good[:20])                                         # shorter than the head
    with pytest.raises(ValueError):
        reopen(good[:-1])                                         # index cut short
    ioff = struct.unpack_from("<Q", good, 16)[0]
    idx = bytearray(good[ioff:])
    # index entry: u16 len, name, u8 code, u8 ndim, u64 dim, u64 off, u64 bytes
    bad = bytearray(idx)
    bad[3] = 5                                                    # unknown dtype code
    with pytest.raises(ValueError):
        reopen(good[:ioff] + bytes(bad))
    bad = bytearray(idx)
    bad[3] = 2                                                    # code disagrees with header
    with pytest.raises(ValueError):
        reopen(good[:ioff] + bytes(bad))
    bad = bytearray(idx)
    struct.pack_into("<Q", bad, 5, C)                             # shape disagrees with header
    with pytest.raises(ValueError):
        reopen(good[:ioff] + bytes(bad))
    bad = bytearray(idx)
    struct.pack_into("<Q", bad, 13, 40)                           # container not 16-aligned
    with pytest.raises(ValueError):
        reopen(good[:ioff] + bytes(bad))
    bad = bytearray(idx)
    struct.pack_into("<Q", bad, 21, ioff)                         # container runs into the index
    with pytest.raises(ValueError):
        reopen(good[:ioff] + bytes(bad))


def test_damaged_counts_and_headers_refused(orc, arc, tmp_path):
    _, cont = _one(orc)
    path = tmp_path / "g.wca"
    arc.write(str(path), [("a", 1, (C + 1,), cont.tobytes())])
    good = bytearray(path.read_bytes())
    ioff = struct.unpack_from("<Q", good, 16)[0]
    for mutate in (lambda b: struct.pack_into("<I", b, 8, 7),      # more entries than the index holds
                   lambda b: b.__setitem__(32, ord("Q"))):          # container magic broken
        bad = bytearray(good)
        mutate(bad)
        p = tmp_path / "bad.wca"
        p.write_bytes(bytes(bad))
        with pytest.raises(ValueError):
            arc.Archive(str(p))
    assert ioff % 16 == 0


def test_checksums_stored_and_read_back(orc, arc, tmp_path):
    ents = _entries(orc)
    block = 8192
    path = str(tmp_path / "c.wca")
    arc.write(path, [(n, c, s, cont.tobytes(), orc.crc32_blocks(cont, block))
                     for n, c, s, _, cont in ents], crc_block=block)
    with arc.Archive(path) as a:
        assert a.crc_block == block
        for name, _, _, _, cont in ents:
            assert np.array_equal(a.container(name), cont)
            assert np.array_equal(a.checksums(name), orc.crc32_blocks(cont, block))
    # a wrong number of checksums is refused when writing
    n, c, s, _, cont = ents[0]
    with pytest.raises(ValueError):
        arc.write(path, [(n, c, s, cont.tobytes(), orc.crc32_blocks(cont, block)[:-1])], crc_block=block)
    with pytest.raises(ValueError):
        arc.write(path, [(n, c, s, cont.tobytes())], crc_block=block)
    # without checksums the list is empty
    arc.write(path, [(n, c, s, cont.tobytes())])
    with arc.Archive(path) as a:
        assert a.crc_block == 0 and a.checksums(n).size == 0


def test_split12_entries(orc, arc, tmp_path):
    """Serving-format (Split12) containers stored beside rANS ones: told apart
    by their magic, checked against the index, checksummed the same way."""
    import split12 as s12
    rng = np.random.default_rng(41)
    b = workloads.rne_bf16(rng.standard_normal(C + 77).astype(np.float32) * np.float32(0.02))
    b[[3, C + 5]] = 0x7A01
    c12 = s12.encode(b)
    crans = orc.encode(b)
    path = str(tmp_path / "s.wca")
    block = 8192
    arc.write(path, [("w12", 1, (C + 77,), c12.tobytes(), orc.crc32_blocks(c12, block)),
                     ("w", 1, (C + 77,), crans.tobytes(), orc.crc32_blocks(crans, block))],
              crc_block=block)
    with arc.Archive(path) as a:
        assert a.codec("w12") == "split12" and a.codec("w") == "rans"
        assert a.info("w12")[:2] == (a.info("w")[0], (C + 77,))
        assert np.array_equal(a.container("w12"), c12)
        assert np.array_equal(s12.decode(a.container("w12")), b)
        assert np.array_equal(a.checksums("w12"), orc.crc32_blocks(c12, block))
    # a Split12 entry must be bf16 and match the index's shape
    for code, shape in ((2, (C + 77,)), (1, (C + 78,))):
        arc.write(path, [("w12", code, shape, c12.tobytes())])
        with pytest.raises(ValueError):
            arc.Archive(path)
    bad = c12.copy()
    bad[20] ^= 1                                                   # chunk count
    arc.write(path, [("w12", 1, (C + 77,), bad.tobytes())])
    with pytest.raises(ValueError):
        arc.Archive(path)
