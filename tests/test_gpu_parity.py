"""GPU parity: containers from the CUDA library are byte-identical to the CPU
oracle's, and decoding is bit-exact, on small and ragged inputs, special
values, single-symbol tables, raw fallback, random access and corrupted
containers.  Everything goes through the C ABI (via the binding)."""
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


@pytest.fixture(scope="module")
def gu():
    import gpu_util
    return gpu_util


def _normal_bits(n, dt, seed, scale=0.02):
    x = np.random.default_rng(seed).standard_normal(n).astype(np.float32) * np.float32(scale)
    return workloads.rne_bf16(x) if dt == "bf16" else x.view(np.uint32).copy()


def _check(orc, gu, bits):
    want = orc.encode(bits)
    got, back = gu.gpu_roundtrip(bits)
    assert got.size == want.size, (got.size, want.size)
    if not np.array_equal(got, want):
        diff = np.nonzero(got != want)[0]
        raise AssertionError(f"{diff.size} bytes differ, first at {diff[:8].tolist()}")
    assert np.array_equal(back, bits)
    return want


def test_workload1_single_tensor(orc, gu):
    bits = workloads.generate_tensor(1, 0)
    _check(orc, gu, bits)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 31, 32, 33, 100, 128, 129, 511, 512, 513,
                               4000, 65535, 65536, 65537, 3 * C + 17, 5 * C + 511])
def test_edge_sizes(orc, gu, dt, n):
    _check(orc, gu, _normal_bits(n, dt, seed=n + 7))


def test_all_bf16_patterns(orc, gu):
    _check(orc, gu, np.arange(1 << 16, dtype=np.uint16))            # raw path
    rng = np.random.default_rng(1)
    base = _normal_bits(16 * C, "bf16", seed=2)
    pos = rng.choice(base.size, size=1 << 16, replace=False)
    base[pos] = np.arange(1 << 16, dtype=np.uint16)
    _check(orc, gu, base)                                            # coded path


def test_fp32_specials(orc, gu):
    sp = np.array([0x00000000, 0x80000000, 0x00000001, 0x807FFFFF, 0x00400000,
                   0x7F800000, 0xFF800000, 0x7F800001, 0xFFC00000, 0x7FFFFFFF,
                   0x7FC00001, 0xFF800001, 0x00800000, 0x7F7FFFFF, 0xFF7FFFFF], np.uint32)
    _check(orc, gu, sp)
    base = _normal_bits(2 * C + 3, "fp32", seed=3)
    base[np.random.default_rng(4).choice(base.size, size=sp.size, replace=False)] = sp
    _check(orc, gu, base)
    rng = np.random.default_rng(5)
    allexp = ((rng.integers(0, 2, 256, dtype=np.uint32) << 31) |
              (np.arange(256, dtype=np.uint32) << 23) | rng.integers(0, 1 << 23, 256, dtype=np.uint32))
    base[:256] = allexp
    _check(orc, gu, base)


def test_single_symbol_and_kinds(orc, gu):
    _check(orc, gu, np.full(3 * C + 5, 0x3C00, np.uint16))
    _check(orc, gu, np.full(200, 0x3F80, np.uint16))
    _check(orc, gu, np.full(C, 0xBF800000, np.uint32))
    for kind in range(4):
        for nch in (1, 3):
            _check(orc, gu, workloads.adversarial_kind_tensor(kind, nch))


def test_normalisation_ties_and_rare_symbols(orc, gu):
    """Tables whose correction step goes both ways, with ties."""
    rng = np.random.default_rng(9)
    # many rare exponents bumped to 1 (d < 0) plus two equal large counts
    e = np.concatenate([np.full(5000, 10), np.full(5000, 20), np.arange(30, 40),
                        rng.integers(0, 256, 300)]).astype(np.uint16)
    rng.shuffle(e)
    _check(orc, gu, (e << 7).astype(np.uint16))
    # d > 0 with tied counts
    _check(orc, gu, (np.array([5, 6, 7] * 1000, np.uint16) << 7).astype(np.uint16))
    # 255 rare symbols + one dominant one
    e = np.concatenate([np.full(1000000, 0), np.arange(1, 256)]).astype(np.uint16)
    _check(orc, gu, ((e << 7) | 0x0001).astype(np.uint16))


def test_random_tables_many_shapes(orc, gu):
    rng = np.random.default_rng(11)
    for trial in range(12):
        n = int(rng.integers(1, 3 * C))
        k = int(rng.integers(1, 40))
        syms = rng.choice(256, size=k, replace=False)
        p = rng.dirichlet(np.full(k, 0.3))
        e = rng.choice(syms, size=n, p=p).astype(np.uint32)
        if trial % 2:
            sm = rng.integers(0, 256, n, dtype=np.uint32)
            bits = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
        else:
            bits = ((rng.integers(0, 2, n, dtype=np.uint32) << 31) | (e << 23) |
                    rng.integers(0, 1 << 23, n, dtype=np.uint32)).astype(np.uint32)
        _check(orc, gu, bits)


def test_decode_chunk_random_access(orc, gu):
    from fp32_weight_compression_b200 import wc
    for dt in ("bf16", "fp32"):
        bits = _normal_bits(4 * C + 999, dt, seed=12)
        cont = orc.encode(bits)
        d = gu.cont_device(cont)
        for k in range(5):
            got = gu.to_bits(wc.decode_chunk(d, k))
            assert np.array_equal(got, bits[k * C:(k + 1) * C])
            assert np.array_equal(got, orc.decode_chunk(cont, k))


def test_decode_of_oracle_containers(orc, gu):
    """The GPU decoder reads containers it did not write."""
    from fp32_weight_compression_b200 import wc
    rng = np.random.Generator(np.random.PCG64([5, 0]))
    bits = workloads._adversarial_chunks(rng, 8)
    cont = orc.encode(bits)
    out = wc.decode(gu.cont_device(cont), shape=(bits.size,), dtype=torch.bfloat16)
    assert np.array_equal(gu.to_bits(out), bits)


def test_batch_api_many_items(orc, gu):
    """300 tensors of mixed sizes and dtypes: more than one launch slice."""
    from fp32_weight_compression_b200 import wc
    rng = np.random.default_rng(13)
    arrs = []
    for i in range(300):
        n = int(rng.choice([0, 1, 7, 100, 1000, C - 3, C + 5]))
        arrs.append(_normal_bits(n, "bf16" if i % 3 else "fp32", seed=100 + i))
    ts = [gu.to_device(a) for a in arrs]
    conts = wc.encode_batch(ts)
    for a, c in zip(arrs, conts):
        assert np.array_equal(c.cpu().numpy(), orc.encode(a))
    outs = wc.decode_batch(conts, [(a.size,) for a in arrs], [t.dtype for t in ts])
    for a, o in zip(arrs, outs):
        assert np.array_equal(gu.to_bits(o), a)


# ---------------------------------------------------------------- corruption
def _decode_status(gu, cont_np, n, dtype, guard=4096):
    """Decode into a buffer with a guard region; returns (status, values, guard intact)."""
    from fp32_weight_compression_b200 import wc
    import ctypes
    elem = 2 if dtype == torch.bfloat16 else 4
    d = gu.cont_device(cont_np)
    buf = torch.full((n * elem + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = wc.load().wc_decode(d.data_ptr(), d.numel(), buf.data_ptr(), n * elem,
                             status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    vals = buf[: n * elem].cpu().numpy()
    vals = vals.view(np.uint16 if elem == 2 else np.uint32)
    intact = bool((buf[n * elem:] == 0xA5).all().item())
    return int(status.item()), vals, intact


def test_corrupt_containers_flagged(orc, gu):
    bits = workloads.generate_tensor(1, 0)[: 2 * C + 1000]
    good = orc.encode(bits)
    n, _, nc = orc.read_header(good)
    st, vals, intact = _decode_status(gu, good, n, torch.bfloat16)
    assert st == 0 and intact and np.array_equal(vals, bits)
    off_exp = int(good[40:48].view(np.uint64)[0])
    mutations = {
        "magic": lambda c: c.__setitem__(0, 0),
        "version": lambda c: c.__setitem__(4, 2),
        "freq sum": lambda c: c[64 + 240:66 + 240].view(np.uint16).__setitem__(0, c[64 + 240:66 + 240].view(np.uint16)[0] + 1),
        "odd length": lambda c: c[576 + 8 * (nc + 1):580 + 8 * (nc + 1)].view(np.uint32).__setitem__(0, c[576 + 8 * (nc + 1):580 + 8 * (nc + 1)].view(np.uint32)[0] + 1),
        "offset": lambda c: c[584:592].view(np.uint64).__setitem__(0, c[584:592].view(np.uint64)[0] + 16),
        "total": lambda c: c[56:64].view(np.uint64).__setitem__(0, c[56:64].view(np.uint64)[0] + 16),
        "state": lambda c: c.__setitem__(off_exp + 5, c[off_exp + 5] ^ 0x40),
    }
    for name, mut in mutations.items():
        c = good.copy()
        mut(c)
        st, vals, intact = _decode_status(gu, c, n, torch.bfloat16)
        assert intact, name
        assert st == 4, (name, st)
        assert orc.decode_status(c)[0] == 4, name
    # truncated container
    st, _, intact = _decode_status(gu, good[:-32], n, torch.bfloat16)
    assert st == 4 and intact
    # too-small output
    from fp32_weight_compression_b200 import wc
    d = gu.cont_device(good)
    buf = torch.full((n * 2 + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert wc.load().wc_decode(d.data_ptr(), d.numel(), buf.data_ptr(), n * 2 - 2,
                               status.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 2 and bool((buf == 0xA5).all().item())


def test_random_flips_never_escape(orc, gu):
    bits = workloads.generate_tensor(1, 0)[: C + 4321]
    good = orc.encode(bits)
    n = bits.size
    rng = np.random.default_rng(21)
    for _ in range(40):
        c = good.copy()
        for _ in range(int(rng.integers(1, 4))):
            c[int(rng.integers(0, c.size))] ^= np.uint8(rng.integers(1, 256))
        st, vals, intact = _decode_status(gu, c, n, torch.bfloat16)
        ost, ovals = orc.decode_status(c)
        assert intact
        assert (st == 0) == (ost == 0), (st, ost)
        if st == 0:
            assert np.array_equal(vals, ovals)


@pytest.mark.parametrize("fmax", [1024, 2047, 2048, 2049, 2964, 4000, 4095])
@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_table_format_boundary(orc, gu, dt, fmax):
    """Exact counts that put the largest frequency at fmax, with several f = 1
    symbols: the coder's narrow table (every f <= 2048) and its wide one on
    both sides of the limit, through the paired-chunk path (4 full chunks)
    and a ragged tail."""
    rng = np.random.default_rng(fmax)
    n = 4 * C                        # f = count / 64 exactly when counts are multiples of 64
    ones = [3, 200, 250][:4096 - fmax]  # f = 1
    rest = 4096 - fmax - len(ones)
    fr = {120: fmax}
    for s in ones:
        fr[s] = 1
    others = [118, 119, 121, 122, 123]
    for i, s in enumerate(others):
        fr[s] = rest // len(others) + (1 if i < rest % len(others) else 0)
    fr = {s: f for s, f in fr.items() if f > 0}
    assert sum(fr.values()) == 4096
    e = np.concatenate([np.full(64 * f, s, np.uint32) for s, f in fr.items()])
    rng.shuffle(e)
    assert e.size == n
    assert np.array_equal(orc.normalize(np.bincount(e, minlength=256).astype(np.uint64)),
                          np.array([fr.get(s, 0) for s in range(256)], np.uint32))
    if dt == "bf16":
        sm = rng.integers(0, 256, n, dtype=np.uint32)
        bits = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    else:
        bits = ((rng.integers(0, 2, n, dtype=np.uint32) << 31) | (e << 23) |
                rng.integers(0, 1 << 23, n, dtype=np.uint32)).astype(np.uint32)
    _check(orc, gu, bits)
    _check(orc, gu, bits[:3 * C + 333])


# ---------------------------------------------------------------- fp16
def _fp16(n, seed, scale=0.02):
    return (np.random.default_rng(seed).standard_normal(n) * scale).astype(np.float16)


def _check16(orc, gu, vals):
    want = orc.encode(vals)
    got, back = gu.gpu_roundtrip(vals)
    assert got.size == want.size and np.array_equal(got, want)
    assert np.array_equal(back.view(np.uint16), vals.view(np.uint16))


@pytest.mark.parametrize("n", [0, 1, 17, 33, 513, 65535, 65536, 65537, 3 * C + 17, 5 * C + 511])
def test_fp16_edge_sizes(orc, gu, n):
    _check16(orc, gu, _fp16(n, seed=n + 3))


def test_fp16_all_patterns(orc, gu):
    pats = np.arange(1 << 16, dtype=np.uint16).view(np.float16)
    _check16(orc, gu, pats)                                          # raw path
    base = _fp16(8 * C, seed=5)
    pos = np.random.default_rng(6).choice(base.size, size=1 << 16, replace=False)
    base[pos] = pats
    _check16(orc, gu, base)                                          # coded path


def test_fp16_single_symbol_and_random_access(orc, gu):
    from fp32_weight_compression_b200 import wc
    _check16(orc, gu, np.full(3 * C + 5, 1.0, np.float16))
    vals = _fp16(4 * C + 999, seed=8)
    cont = orc.encode(vals)
    d = gu.cont_device(cont)
    for k in range(5):
        got = wc.decode_chunk(d, k).view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, vals.view(np.uint16)[k * C:(k + 1) * C])


def test_mixed_dtype_batch(orc, gu):
    """bf16, fp16 and fp32 tensors in one batched launch."""
    from fp32_weight_compression_b200 import wc
    arrs = [_normal_bits(2 * C + 7, "bf16", seed=1), _fp16(3 * C + 1, seed=2),
            _normal_bits(C + 5, "fp32", seed=3), _fp16(100, seed=4), _fp16(2 * C, seed=5)]
    ts = [gu.to_device(a) for a in arrs]
    conts = wc.encode_batch(ts)
    for a, c in zip(arrs, conts):
        assert np.array_equal(c.cpu().numpy(), orc.encode(a))
    outs = wc.decode_batch(conts, [(a.size,) for a in arrs], [t.dtype for t in ts])
    for a, o in zip(arrs, outs):
        assert np.array_equal(gu.to_bits(o).view(a.dtype), a)


# ---------------------------------------------------------------- fp8 e4m3
def _fp8(n, seed):
    """Bits of e4m3 values with a weight-like skew: exponents around 6."""
    rng = np.random.default_rng(seed)
    e = np.clip(rng.normal(6, 1.3, n), 0, 15).astype(np.int64)
    return ((rng.integers(0, 2, n) << 7) | (e << 3) | rng.integers(0, 8, n)).astype(np.uint8)


def _check8(orc, gu, bits):
    want = orc.encode(bits)
    got, back = gu.gpu_roundtrip(bits)
    assert got.size == want.size and np.array_equal(got, want)
    assert np.array_equal(back, bits)


@pytest.mark.parametrize("n", [0, 1, 2, 3, 15, 16, 17, 33, 511, 513, 65535, 65536, 65537,
                               3 * C + 17, 5 * C + 511])
def test_fp8_edge_sizes(orc, gu, n):
    _check8(orc, gu, _fp8(n, seed=n + 11))


def test_fp8_all_patterns_and_kinds(orc, gu):
    pats = np.arange(256, dtype=np.uint8)
    _check8(orc, gu, np.tile(pats, 300))                           # near-uniform: raw chunks
    base = _fp8(4 * C + 3, seed=12)
    base[np.random.default_rng(13).choice(base.size, 256, replace=False)] = pats
    _check8(orc, gu, base)                                        # coded with every pattern
    _check8(orc, gu, np.full(2 * C + 9, 0x38, np.uint8))           # single symbol


def test_fp8_random_access_and_mixed_batch(orc, gu):
    from fp32_weight_compression_b200 import wc
    bits = _fp8(4 * C + 999, seed=14)
    d = gu.cont_device(orc.encode(bits))
    for k in range(5):
        got = wc.decode_chunk(d, k).view(torch.uint8).cpu().numpy()
        assert np.array_equal(got, bits[k * C:(k + 1) * C])
    arrs = [_fp8(2 * C + 7, 15), _normal_bits(C + 3, "bf16", 16), _fp8(101, 17), _fp16(C, 18),
            _normal_bits(77, "fp32", 19), _fp8(3 * C, 20)]
    ts = [gu.to_device(a) for a in arrs]
    conts = wc.encode_batch(ts)
    for a, c in zip(arrs, conts):
        assert np.array_equal(c.cpu().numpy(), orc.encode(a))
    outs = wc.decode_batch(conts, [(a.size,) for a in arrs], [t.dtype for t in ts])
    for a, o in zip(arrs, outs):
        assert np.array_equal(gu.to_bits(o).view(a.dtype), a)


@pytest.mark.parametrize("fname,raw", [("container_bf16_n186_tie_raw.txt", True),
                                       ("container_bf16_n186_near_coded.txt", False)])
def test_raw_fallback_boundary(orc, gu, fname, raw):
    """128 + 2w == nsym is stored raw, 128 + 2w == nsym - 2 stays coded:
    the library's container equals the hand-laid-out fixture (and the
    oracle's), and decodes bit-exactly."""
    from _golden import load_container, load_fields
    e = np.array(load_fields(fname)["exponents"], np.uint16)
    bits = (e << 7).astype(np.uint16)
    want = load_container(fname)
    got = _check(orc, gu, bits)
    assert np.array_equal(got, want)
    assert int(want[592:596].view(np.uint32)[0]) == (186 if raw else 184)


# fp8 e5m2 (dtype 5): the coded nibble is exponent bits 4..1, the raw nibble
# exponent bit 0, sign and mantissa ("PTWM", Supported dtypes, float8_e5m2).
def _e5m2(n, seed):
    """Bits of e5m2 values with a weight-like skew: exponents around 12."""
    rng = np.random.default_rng(seed)
    e = np.clip(rng.normal(12, 2.0, n), 0, 31).astype(np.int64)
    return ((rng.integers(0, 2, n) << 7) | (e << 2) | rng.integers(0, 4, n)).astype(np.uint8)


def _check5(orc, gu, bits):
    want = orc.encode(bits, dtype=orc.FP8E5M2)
    got, back = gu.gpu_roundtrip(bits, torch.float8_e5m2)
    assert got.size == want.size and np.array_equal(got, want)
    assert np.array_equal(back, bits)
    return want


@pytest.mark.parametrize("n", [0, 1, 2, 3, 15, 16, 17, 33, 511, 513, 65535, 65536, 65537,
                               3 * C + 17, 5 * C + 511])
def test_fp8e5m2_edge_sizes(orc, gu, n):
    _check5(orc, gu, _e5m2(n, seed=n + 21))


def test_fp8e5m2_all_patterns_and_kinds(orc, gu):
    pats = np.arange(256, dtype=np.uint8)
    _check5(orc, gu, np.tile(pats, 300))                           # near-uniform: raw chunks
    base = _e5m2(4 * C + 3, seed=22)
    base[np.random.default_rng(23).choice(base.size, 256, replace=False)] = pats
    _check5(orc, gu, base)                                        # coded with every pattern
    _check5(orc, gu, np.full(2 * C + 9, 0x3C, np.uint8))           # single symbol
    # the golden hand-derived container
    from _golden import load_container
    want = load_container("container_fp8e5m2_n4_raw.txt")
    got = _check5(orc, gu, np.array([0x3C, 0x3C, 0x3C, 0x38], np.uint8))
    assert np.array_equal(got, want)


def test_fp8e5m2_random_access_and_mixed_batch(orc, gu):
    from fp32_weight_compression_b200 import wc
    bits = _e5m2(4 * C + 999, seed=24)
    d = gu.cont_device(orc.encode(bits, dtype=orc.FP8E5M2))
    for k in range(5):
        got = wc.decode_chunk(d, k).view(torch.uint8).cpu().numpy()
        assert np.array_equal(got, bits[k * C:(k + 1) * C])
    arrs = [_e5m2(2 * C + 7, 25), _fp8(C + 3, 26), _e5m2(101, 27), _normal_bits(77, "bf16", 28)]
    fp8s = [torch.float8_e5m2, torch.float8_e4m3fn, torch.float8_e5m2, None]
    ts = [gu.to_device(a, f) if f is not None else gu.to_device(a) for a, f in zip(arrs, fp8s)]
    conts = wc.encode_batch(ts)
    for a, f, c in zip(arrs, fp8s, conts):
        want = orc.encode(a, dtype=orc.FP8E5M2) if f == torch.float8_e5m2 else orc.encode(a)
        assert np.array_equal(c.cpu().numpy(), want)
    outs = wc.decode_batch(conts, [(a.size,) for a in arrs], [t.dtype for t in ts])
    for a, o in zip(arrs, outs):
        assert np.array_equal(gu.to_bits(o).view(a.dtype), a)
