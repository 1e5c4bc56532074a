"""Oracle round trips (bit-exact), edge sizes, special values, random access
and corrupted containers.  No GPU needed."""
import numpy as np
import pytest

import workloads

C = 65536


def _skewed_with(patterns: np.ndarray, nchunks: int, seed: int, dtype=np.uint16) -> np.ndarray:
    """Spread `patterns` over nchunks chunks of N(0, 0.02) data so that every
    chunk stays compressible (coded) while containing the given bit patterns."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(nchunks * C).astype(np.float32) * np.float32(0.02)
    if dtype == np.uint16:
        base = workloads.rne_bf16(x)
    else:
        base = x.view(np.uint32).copy()
    pos = rng.choice(base.size, size=patterns.size, replace=False)
    base[pos] = patterns
    return base


def test_all_bf16_patterns_raw_path(orc):
    bits = np.arange(1 << 16, dtype=np.uint16)
    cont = orc.encode(bits)
    assert np.array_equal(orc.decode(cont), bits)
    # uniform exponents cannot shrink: the chunk is raw
    n, dt, nc = orc.read_header(cont)
    assert nc == 1 and int(cont[576 + 16:576 + 20].view(np.uint32)[0]) == C


def test_all_bf16_patterns_coded_path(orc):
    bits = _skewed_with(np.arange(1 << 16, dtype=np.uint16), 16, seed=1)
    cont = orc.encode(bits)
    n, dt, nc = orc.read_header(cont)
    lens = cont[576 + 8 * (nc + 1): 576 + 8 * (nc + 1) + 4 * nc].view(np.uint32)
    assert np.all(lens < C)  # every chunk coded
    assert np.array_equal(orc.decode(cont), bits)


FP32_SPECIALS = np.array([
    0x00000000, 0x80000000,                 # +-0
    0x00000001, 0x807FFFFF, 0x00400000,     # subnormals
    0x7F800000, 0xFF800000,                 # +-Inf
    0x7F800001, 0xFFC00000, 0x7FFFFFFF,     # sNaN / qNaN payloads
    0x7FC00001, 0xFF800001,
    0x00800000, 0x7F7FFFFF, 0xFF7FFFFF,     # smallest normal, +-max
], dtype=np.uint32)


def test_fp32_special_values(orc):
    bits = _skewed_with(FP32_SPECIALS, 1, seed=2, dtype=np.uint32)
    cont = orc.encode(bits)
    assert np.array_equal(orc.decode(cont), bits)
    # the specials alone (raw path)
    cont = orc.encode(FP32_SPECIALS)
    assert np.array_equal(orc.decode(cont), FP32_SPECIALS)


def test_fp32_every_exponent(orc):
    rng = np.random.default_rng(3)
    e = np.arange(256, dtype=np.uint32)
    m = rng.integers(0, 1 << 23, size=256, dtype=np.uint32)
    s = rng.integers(0, 2, size=256, dtype=np.uint32)
    pats = (s << 31) | (e << 23) | m
    bits = _skewed_with(pats, 2, seed=4, dtype=np.uint32)
    cont = orc.encode(bits)
    assert np.array_equal(orc.decode(cont), bits)


@pytest.mark.parametrize("n", [0, 1, 31, 32, 33, 100, 128, 129, 65535, 65536, 65537, 3 * C + 17])
@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_edge_sizes(orc, n, dt):
    rng = np.random.default_rng(n)
    x = (rng.standard_normal(n).astype(np.float32) * np.float32(0.02))
    bits = workloads.rne_bf16(x) if dt == "bf16" else x.view(np.uint32).copy()
    cont = orc.encode(bits)
    assert cont.size <= orc.encode_bound(n, 1 if dt == "bf16" else 2)
    assert cont.size % 16 == 0
    assert np.array_equal(orc.decode(cont), bits)
    n2, _, nc = orc.read_header(cont)
    assert n2 == n and nc == (n + C - 1) // C
    for k in range(nc):
        assert np.array_equal(orc.decode_chunk(cont, k), bits[k * C:(k + 1) * C])


def test_single_symbol_tensor(orc):
    bits = np.full(3 * C + 5, 0x3C00, np.uint16)
    cont = orc.encode(bits)
    f = cont[64:576].view(np.uint16)
    assert f[0x3C00 >> 7] == 4096 and int(f.sum()) == 4096
    n, dt, nc = orc.read_header(cont)
    lens = cont[576 + 8 * (nc + 1): 576 + 8 * (nc + 1) + 4 * nc].view(np.uint32)
    assert lens.tolist() == [128, 128, 128, 5]  # last chunk: 128 >= 5 -> raw
    assert np.array_equal(orc.decode(cont), bits)


def test_adversarial_kinds_round_trip(orc):
    for kind in range(4):
        bits = workloads.adversarial_kind_tensor(kind, 2)
        cont = orc.encode(bits)
        assert np.array_equal(orc.decode(cont), bits)
        n, dt, nc = orc.read_header(cont)
        lens = cont[576 + 8 * (nc + 1): 576 + 8 * (nc + 1) + 4 * nc].view(np.uint32)
        if kind == 0:
            assert np.all(lens == C)       # incompressible -> raw fallback
        if kind in (1, 3):
            assert np.all(lens < C)        # single symbol / skewed -> coded


def test_mixed_adversarial_stream(orc):
    rng = np.random.Generator(np.random.PCG64([5, 0]))
    bits = workloads._adversarial_chunks(rng, 8)
    cont = orc.encode(bits)
    assert np.array_equal(orc.decode(cont), bits)


# ---------------------------------------------------------------- corruption
def _good():
    bits = workloads.generate_tensor(1, 0)[: 2 * C + 1000]
    return bits


def _field(cont, off, dt):
    return cont[off:off + np.dtype(dt).itemsize].view(dt)


def test_corrupt_header_fields(orc):
    bits = _good()
    good = orc.encode(bits)
    n, dt, nc = orc.read_header(good)
    cases = []
    c = good.copy(); c[0] ^= 1; cases.append(c)                       # magic
    c = good.copy(); c[4] = 2; cases.append(c)                        # version
    c = good.copy(); c[6] = 7; cases.append(c)                        # dtype (unknown)
    c = good.copy(); c[7] = 16; cases.append(c)                       # lanes
    c = good.copy(); _field(c, 16, np.uint32)[0] = 4096; cases.append(c)
    c = good.copy(); _field(c, 24, np.uint16)[0] = 11; cases.append(c)
    c = good.copy(); _field(c, 64 + 2 * 120, np.uint16)[0] += 1; cases.append(c)  # freq sum
    c = good.copy(); _field(c, 576 + 8 * (nc + 1), np.uint32)[0] += 1; cases.append(c)  # odd length
    c = good.copy(); _field(c, 576 + 8 * (nc + 1), np.uint32)[0] = C + 1; cases.append(c)
    c = good.copy(); _field(c, 576 + 8, np.uint64)[0] += 16; cases.append(c)  # offsets
    c = good.copy(); _field(c, 56, np.uint64)[0] += 16; cases.append(c)  # total
    c = good[:-16].copy(); cases.append(c)                            # truncated
    c = good[:100].copy(); cases.append(c)
    for i, cc in enumerate(cases):
        st, _ = orc.decode_status(cc)
        assert st == 4, f"case {i} not rejected"


def test_corrupt_words_detected(orc):
    bits = _good()
    good = orc.encode(bits)
    off_exp = int(_field(good, 40, np.uint64)[0])
    c = good.copy()
    c[off_exp + 128 + 500] ^= 0x5A   # inside chunk 0's words
    st, out = orc.decode_status(c)
    # a flipped word either breaks the final-state check or changes the output
    assert st == 4 or not np.array_equal(out, bits)
    c = good.copy()
    c[off_exp + 3] ^= 0x01           # a final state
    st, out = orc.decode_status(c)
    assert st == 4 or not np.array_equal(out, bits)


def test_random_byte_flips_never_crash(orc):
    bits = _good()
    good = orc.encode(bits)
    rng = np.random.default_rng(11)
    for _ in range(300):
        c = good.copy()
        for _ in range(int(rng.integers(1, 4))):
            c[int(rng.integers(0, c.size))] ^= np.uint8(rng.integers(1, 256))
        st, _ = orc.decode_status(c)
        assert st in (0, 4)
