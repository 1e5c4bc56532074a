"""The fused Split12 linear layer on the GPU (wc12_linear through the C ABI):
Y = X W^T with W held as a Split12 container ("weight-compression" README:
bf16 weights rebuilt from a codebook index and the raw low byte inside the
serving kernels), against the oracle's float64 sum of the exact bf16
products (oracle/split12.py linear): TMA loads, the weights expanded into
the tensor cores' operand layout, tcgen05 MMAs.

Tolerance, from the arithmetic: every product of two bf16 values is exact in
fp32, so an output is a sum of K exact terms; the tensor cores and the split-K
atomics add them in fp32 in some order, at most m = K + K/64 additions, each
off by at most one unit in the last place of its result (relative 2^-23,
which also covers rounding toward zero).  The classic bound on such a sum is
|y - y64| <= gamma_m * sum|x w| with gamma_m = m u / (1 - m u), u = 2^-23.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp32_weight_compression_b200 import build
    build.build()


@pytest.fixture(scope="module")
def s12():
    import split12
    return split12


def _bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda")


def _to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def _weights(N, K, seed, outliers=0.0):
    """bf16 weights: N(0, 0.02), with a fraction of outliers whose high bytes
    are spread over many rare values (so they become exceptions)."""
    rng = np.random.default_rng(seed)
    w = workloads.rne_bf16(rng.standard_normal(N * K).astype(np.float32) * np.float32(0.02))
    if outliers > 0:
        m = rng.random(N * K) < outliers
        mag = np.float32(2.0) ** rng.integers(-20, 12, int(m.sum())).astype(np.float32)
        sgn = np.where(rng.random(int(m.sum())) < 0.5, -1.0, 1.0).astype(np.float32)
        w[m] = workloads.rne_bf16(mag * sgn * np.float32(1.5))
    return w


def _check(s12, N, K, M, seed, outliers=0.0):
    from fp32_weight_compression_b200 import wc
    wbits = _weights(N, K, seed, outliers)
    cont = s12.encode(wbits)
    rng = np.random.default_rng(seed + 1)
    xbits = workloads.rne_bf16(rng.standard_normal(M * K).astype(np.float32))
    y64 = s12.linear(xbits.reshape(M, K), cont, N)
    absum = np.abs(_to_f64(xbits).reshape(M, K)) @ np.abs(_to_f64(wbits).reshape(N, K)).T
    dcont = torch.from_numpy(cont).to("cuda")
    y = wc.split12_linear(dcont, N, K, _bf16_dev(xbits).view(M, K))
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    m = K + K // 64  # K products and at most one split-K atomic per 64-value stage
    u = 2.0 ** -23
    gamma = m * u / (1 - m * u)
    err = np.abs(got - y64)
    bound = gamma * absum
    bad = np.nonzero(err > bound)
    assert bad[0].size == 0, (f"{bad[0].size} outputs off; first (token, row) "
                              f"{bad[0][0]}, {bad[1][0]}: {got[bad][0]} vs {y64[bad][0]}")
    return s12.read_header(cont)["ne"]


def test_one_small_shape_first(s12):
    _check(s12, 128, 64, 1, seed=1)


@pytest.mark.parametrize("N,K", [(128, 64), (256, 128), (128, 4096), (256, 4096)])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 144, 256, 300])
def test_shapes(s12, N, K, M):
    _check(s12, N, K, M, seed=N + K + M)


@pytest.mark.parametrize("K", [64, 4096])
def test_exceptions_in_the_tile(s12, K):
    """Outliers become exceptions: a few per tile (gathered into the CTA's
    list) and, at 20 %, more than the list holds (walked per stage)."""
    for frac in (0.002, 0.2):
        for M in (1, 4, 33):
            ne = _check(s12, 256, K, M, seed=K + int(frac * 1000) + M, outliers=frac)
            assert ne > 0


def test_corrupt_header_is_reported(s12):
    from fp32_weight_compression_b200 import wc
    N, K = 128, 128
    cont = s12.encode(_weights(N, K, 3))
    for M in (1, 17):
        x = _bf16_dev(workloads.rne_bf16(np.ones(M * K, np.float32))).view(M, K)
        for off, val in ((0, 0x00), (8, 0x01), (16, 0x00)):   # magic, n, chunk size
            bad = cont.copy()
            bad[off] ^= 0xFF if val == 0 else val
            with pytest.raises(wc.WCError) as ei:
                wc.split12_linear(torch.from_numpy(bad).to("cuda"), N, K, x)
            assert ei.value.code == wc.ERR_CORRUPT
        # the intact container still works after the refusals
        y = wc.split12_linear(torch.from_numpy(cont).to("cuda"), N, K, x)
        assert torch.isfinite(y).all()


def test_short_buffer_is_refused(s12):
    """A buffer that cannot hold the index and low planes of an N x K
    container is refused before any launch."""
    from fp32_weight_compression_b200 import wc
    N, K = 128, 256
    cont = s12.encode(_weights(N, K, 5))
    short = torch.from_numpy(cont[:N * K]).to("cuda")  # header + index plane, not all low bytes
    for M in (1, 2, 40):
        x = _bf16_dev(workloads.rne_bf16(np.ones(M * K, np.float32))).view(M, K)
        with pytest.raises(wc.WCError) as ei:
            wc.split12_linear(short, N, K, x)
        assert ei.value.code == wc.ERR_INVALID_ARG
