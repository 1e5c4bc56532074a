"""The archive file on the GPU: save() writes the library's containers (byte
for byte the oracle's) under their names, and load / load_chunk / load_all
give the tensors back bit-exact."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu
C = 65536


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp32_weight_compression_b200 import build
    build.build()


def _tensors():
    import gpu_util as gu
    rng = np.random.default_rng(21)
    bf = workloads.rne_bf16(rng.standard_normal(3 * C + 6).astype(np.float32) * np.float32(0.02))
    f32 = (rng.standard_normal(2 * C + 1).astype(np.float32) * np.float32(0.02)).view(np.uint32)
    f16 = (rng.standard_normal(C + 77) * 0.05).astype(np.float16)
    e = np.clip(rng.normal(6, 1.3, 2 * C + 9), 0, 15).astype(np.int64)
    f8 = ((rng.integers(0, 2, e.size) << 7) | (e << 3) | rng.integers(0, 8, e.size)).astype(np.uint8)
    bits = {"blk.0.attn.q": (bf, (6, 32769)), "norm": (f32, (2 * C + 1,)),
            "h16": (f16, (C + 77, 1)), "f8": (f8, (2 * C + 9,)), "none": (np.zeros(0, np.uint16), (0,))}
    return {k: (b, gu.to_device(b).reshape(s)) for k, (b, s) in bits.items()}


def test_save_load_bit_exact(orc, tmp_path):
    import gpu_util as gu
    from fp32_weight_compression_b200 import archive
    ts = _tensors()
    path = str(tmp_path / "m.wca")
    archive.save(path, {k: t for k, (_, t) in ts.items()})
    with archive.Archive(path) as a:
        assert a.names() == list(ts)
        for k, (b, t) in ts.items():
            assert a.info(k)[:2] == (t.dtype, tuple(t.shape))
            assert np.array_equal(a.container(k), orc.encode(b))
            got = a.load(k)
            assert got.dtype == t.dtype and tuple(got.shape) == tuple(t.shape)
            assert np.array_equal(gu.to_bits(got).reshape(-1).view(np.uint8), b.view(np.uint8))
        # one chunk: the second of the bf16 tensor and the ragged last of fp8
        part = a.load_chunk("blk.0.attn.q", 1)
        assert np.array_equal(gu.to_bits(part), ts["blk.0.attn.q"][0][C:2 * C])
        part = a.load_chunk("f8", 2)
        assert np.array_equal(gu.to_bits(part), ts["f8"][0][2 * C:])
        for k in range(3):   # fp32 (sign-bit and mantissa ranges), and without checks
            part = a.load_chunk("norm", k, verify=k != 1)
            assert np.array_equal(gu.to_bits(part), ts["norm"][0][k * C:(k + 1) * C])
        allv = a.load_all()
        for k, (b, t) in ts.items():
            assert allv[k].dtype == t.dtype and tuple(allv[k].shape) == tuple(t.shape)
            assert np.array_equal(gu.to_bits(allv[k]).reshape(-1).view(np.uint8), b.view(np.uint8))
        some = a.load_all(["h16", "norm"])
        assert list(some) == ["h16", "norm"]


def test_checksums_catch_a_damaged_container(orc, tmp_path):
    import gpu_util as gu
    from fp32_weight_compression_b200 import archive
    ts = _tensors()
    path = tmp_path / "c.wca"
    block = 65536
    archive.save(str(path), {k: t for k, (_, t) in ts.items()}, crc_block=block)
    with archive.Archive(str(path)) as a:
        assert a.crc_block == block
        for k in ts:
            assert np.array_equal(a.checksums(k), orc.crc32_blocks(a.container(k), block))
            assert a.verify(k) == []
        off = a._entries["blk.0.attn.q"][2]
        size = a.info("blk.0.attn.q")[2]
    # flip one bit in the second checksum block of that container
    raw = bytearray(path.read_bytes())
    pos = off + block + 1234
    assert pos < off + size
    raw[pos] ^= 0x04
    path.write_bytes(bytes(raw))
    with archive.Archive(str(path)) as a:
        assert a.verify("blk.0.attn.q") == [1]
        with pytest.raises(ValueError):
            a.load("blk.0.attn.q")
        with pytest.raises(ValueError):
            a.load_all()
        # one chunk: its bytes include the damaged block (chunk 0's raw plane
        # reaches into checksum block 1) or do not (chunk 2)
        with pytest.raises(ValueError):
            a.load_chunk("blk.0.attn.q", 0)
        part = a.load_chunk("blk.0.attn.q", 2)
        assert np.array_equal(gu.to_bits(part), ts["blk.0.attn.q"][0][2 * C:3 * C])
        # the other entries are untouched
        got = a.load("h16")
        assert np.array_equal(gu.to_bits(got).reshape(-1), ts["h16"][0])


def test_split12_archive(orc, tmp_path):
    import gpu_util as gu
    import split12 as s12
    from fp32_weight_compression_b200 import archive
    ts = _tensors()
    bf = {k: v for k, v in ts.items() if v[1].dtype == torch.bfloat16}
    path = str(tmp_path / "serve.wca")
    archive.save(path, {k: t for k, (_, t) in bf.items()}, codec="split12", crc_block=65536)
    with archive.Archive(path) as a:
        for k, (b, t) in bf.items():
            assert a.codec(k) == "split12"
            assert np.array_equal(a.container(k), s12.encode(b))
            assert a.verify(k) == []
            got = a.load(k)
            assert got.dtype == torch.bfloat16 and tuple(got.shape) == tuple(t.shape)
            assert np.array_equal(gu.to_bits(got).reshape(-1), b)
            dc = a.device_container(k)
            assert dc.is_cuda and np.array_equal(dc.cpu().numpy(), a.container(k))
        allv = a.load_all()
        for k, (b, t) in bf.items():
            assert np.array_equal(gu.to_bits(allv[k]).reshape(-1), b)
        with pytest.raises(ValueError):
            a.load_chunk(next(iter(bf)), 0)
