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
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 64, 144, 200, 256, 300])
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


def _plan_from_oracle(s12, cont, N, K):
    """The serving plan's starts and (per bucket, sorted) entries, built from
    the container's exception lists in numpy: the definition the GPU plan
    must meet (its order within a bucket is free)."""
    h = s12.read_header(cont)
    lay = s12.layout(h["n"], h["ne"])
    nc = lay["nc"]
    exc_off = np.frombuffer(cont[80:80 + 8 * (nc + 1)].tobytes(), np.uint64).astype(np.int64)
    pos = np.frombuffer(cont[lay["off_exc"]:lay["off_exc"] + 2 * h["ne"]].tobytes(), np.uint16).astype(np.int64)
    hi = cont[lay["off_excval"]:lay["off_excval"] + h["ne"]].astype(np.int64)
    chunk = np.repeat(np.arange(nc), np.diff(exc_off))
    f = chunk * 65536 + pos
    row, col = f // K, f % K
    S = K // 64
    bucket = (row // 128) * S + col // 64
    entry = (col % 64) | ((row % 128) << 6) | (hi << 16)
    nb = (N // 128) * S
    counts = np.bincount(bucket, minlength=nb)
    starts = np.concatenate([[0], np.cumsum(counts)])
    per = [np.sort(entry[bucket == b]) for b in range(nb)]
    return h["ne"], starts, per


@pytest.mark.parametrize("N,K,outliers", [(128, 64, 0.0), (256, 4096, 0.002), (384, 1024, 0.2)])
def test_plan_matches_its_definition(s12, N, K, outliers):
    from fp32_weight_compression_b200 import wc
    cont = s12.encode(_weights(N, K, 21, outliers))
    ne, starts, per = _plan_from_oracle(s12, cont, N, K)
    plan = wc.split12_plan(torch.from_numpy(cont).to("cuda"), N, K).cpu().numpy()
    assert plan.size == wc.split12_plan_bytes(N, K, ne)
    h = np.frombuffer(plan[:32].tobytes(), np.uint32)
    assert tuple(h[:4]) == (0x50323157, 1, N, K)
    nb = (N // 128) * (K // 64)
    assert tuple(np.frombuffer(plan[16:32].tobytes(), np.uint64)) == (ne, nb)
    got_starts = np.frombuffer(plan[32:32 + 4 * (nb + 1)].tobytes(), np.uint32).astype(np.int64)
    assert np.array_equal(got_starts, starts)
    off_ent = (32 + 4 * (nb + 1) + 15) // 16 * 16
    ent = np.frombuffer(plan[off_ent:off_ent + 4 * ne].tobytes(), np.uint32).astype(np.int64)
    for b in range(nb):
        assert np.array_equal(np.sort(ent[starts[b]:starts[b + 1]]), per[b]), b


@pytest.mark.parametrize("N,K", [(128, 64), (256, 128), (128, 4096), (256, 4096)])
@pytest.mark.parametrize("M", [1, 2, 16, 17, 64, 144, 256, 300])
def test_planned_shapes(s12, N, K, M):
    _check_planned(s12, N, K, M, seed=N + K + M + 7)


def _check_planned(s12, N, K, M, seed, outliers=0.0):
    from fp32_weight_compression_b200 import wc
    wbits = _weights(N, K, seed, outliers)
    cont = s12.encode(wbits)
    rng = np.random.default_rng(seed + 1)
    xbits = workloads.rne_bf16(rng.standard_normal(M * K).astype(np.float32))
    y64 = s12.linear(xbits.reshape(M, K), cont, N)
    absum = np.abs(_to_f64(xbits).reshape(M, K)) @ np.abs(_to_f64(wbits).reshape(N, K)).T
    dcont = torch.from_numpy(cont).to("cuda")
    plan = wc.split12_plan(dcont, N, K)
    y = wc.split12_linear(dcont, N, K, _bf16_dev(xbits).view(M, K), plan=plan)
    torch.cuda.synchronize()
    m = K + K // 64
    u = 2.0 ** -23
    bound = m * u / (1 - m * u) * absum
    err = np.abs(y.cpu().numpy().astype(np.float64) - y64)
    assert (err <= bound).all(), int((err > bound).sum())
    # the same bits as without the plan, up to the split-K atomics' order
    y0 = wc.split12_linear(dcont, N, K, _bf16_dev(xbits).view(M, K))
    assert (np.abs(y0.cpu().numpy().astype(np.float64) - y64) <= bound).all()


@pytest.mark.parametrize("K", [64, 4096])
def test_planned_exceptions(s12, K):
    """1 in 500 values an exception (the plan's range copied to shared
    memory) and 1 in 5 (more than a CTA's list holds: read at each stage)."""
    for frac in (0.002, 0.2):
        for M in (1, 33):
            _check_planned(s12, 256, K, M, seed=K + int(frac * 1000) + M + 3, outliers=frac)


def test_plan_mismatch_and_corruption_are_reported(s12):
    from fp32_weight_compression_b200 import wc
    N, K = 128, 256
    cont = s12.encode(_weights(N, K, 8, 0.01))
    other = s12.encode(_weights(N, K, 9, 0.03))
    dcont, dother = torch.from_numpy(cont).to("cuda"), torch.from_numpy(other).to("cuda")
    plan = wc.split12_plan(dcont, N, K)
    x = _bf16_dev(workloads.rne_bf16(np.ones(4 * K, np.float32))).view(4, K)
    # a plan built for another container (another exception count)
    assert s12.read_header(cont)["ne"] != s12.read_header(other)["ne"]
    with pytest.raises(wc.WCError) as ei:
        wc.split12_linear(dother, N, K, x, plan=plan)
    assert ei.value.code == wc.ERR_CORRUPT
    # a plan whose header (magic, N) was damaged, or whose starts run past
    # the exception count or out of order (a plan is an index, not a
    # checksummed copy: damage that keeps the starts in order goes unseen)
    for off, val in ((0, 0xFF), (8, 0x01)):
        bad = plan.clone()
        bad[off] ^= val
        with pytest.raises(wc.WCError) as ei:
            wc.split12_linear(dcont, N, K, x, plan=bad)
        assert ei.value.code == wc.ERR_CORRUPT
    for i, v in ((1, 0xFFFFFFFF), (4, 0)):
        bad = plan.clone()
        bad[32 + 4 * i:32 + 4 * i + 4] = torch.tensor(list(int(v).to_bytes(4, "little")), dtype=torch.uint8)
        with pytest.raises(wc.WCError) as ei:
            wc.split12_linear(dcont, N, K, x, plan=bad)
        assert ei.value.code == wc.ERR_CORRUPT
    # a plan too short for its starts is refused on the host
    with pytest.raises(wc.WCError) as ei:
        wc.split12_linear(dcont, N, K, x, plan=plan[:40])
    assert ei.value.code == wc.ERR_INVALID_ARG
    # a corrupt container yields an invalid plan, which is then refused
    badc = cont.copy()
    h = s12.read_header(cont)
    lay = s12.layout(h["n"], h["ne"])
    badc[lay["off_exc"]:lay["off_exc"] + 2] = 0xFF  # first exception position past its chunk
    with pytest.raises(wc.WCError) as ei:
        wc.split12_plan(torch.from_numpy(badc).to("cuda"), N, K)
    assert ei.value.code == wc.ERR_CORRUPT
    # the intact pair still works
    y = wc.split12_linear(dcont, N, K, x, plan=plan)
    assert torch.isfinite(y).all()
