"""Block checksums on the GPU (wc_crc32_blocks) against the oracle's bitwise
CRC-32: ragged sizes and tails, several block sizes, constant buffers, a
flipped bit, and a buffer of many blocks."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp32_weight_compression_b200 import build
    build.build()


def _gpu(data: np.ndarray, block: int) -> np.ndarray:
    from fp32_weight_compression_b200 import wc
    d = torch.from_numpy(data).to("cuda")
    out = wc.crc32_blocks(d, block)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 15, 16, 17, 63, 64, 65, 8191, 8192, 8193,
                               3 * 8192 + 77, (1 << 20) - 1, 1 << 20, (1 << 20) + 1,
                               3 * (1 << 20) + 12345])
@pytest.mark.parametrize("block", [8192, 65536, 1 << 20])
def test_matches_oracle(orc, n, block):
    data = np.random.default_rng(n + block).integers(0, 256, n, dtype=np.uint8)
    assert np.array_equal(_gpu(data, block), orc.crc32_blocks(data, block))


def test_constant_buffers_and_a_flipped_bit(orc):
    n, block = 5 * 65536 + 3, 65536
    for v in (0, 0xFF):
        data = np.full(n, v, np.uint8)
        assert np.array_equal(_gpu(data, block), orc.crc32_blocks(data, block))
    data = np.random.default_rng(4).integers(0, 256, n, dtype=np.uint8)
    good = _gpu(data, block)
    data[2 * 65536 + 999] ^= 0x10
    bad = _gpu(data, block)
    assert np.array_equal(bad, orc.crc32_blocks(data, block))
    assert np.nonzero(bad != good)[0].tolist() == [2]


def test_many_blocks(orc):
    # more blocks than resident CTAs: every CTA loops over several blocks
    n, block = 600 * 65536 + 4321, 65536
    data = np.random.default_rng(6).integers(0, 256, n, dtype=np.uint8)
    assert np.array_equal(_gpu(data, block), orc.crc32_blocks(data, block))


def test_largest_block(orc):
    # one short block of the largest size: 2 MiB per thread, most threads idle
    n, block = (64 << 20) + 5, 1 << 30
    data = np.random.default_rng(7).integers(0, 256, n, dtype=np.uint8)
    assert np.array_equal(_gpu(data, block), orc.crc32_blocks(data, block))
