"""Pins of the CPU oracle against things other than itself: hand-worked traces
and containers (tests/golden/), normalisation examples worked by hand, brute
force over tiny inputs, the exact rANS accounting bound, and information
theory.  No GPU needed."""
import itertools

import numpy as np
import pytest

from _golden import load_container, load_traces

L = 65536


# ---------------------------------------------------------------- traces
@pytest.mark.parametrize("name", ["T1", "T2", "T3"])
def test_hand_traces(orc, name):
    tr = load_traces()[name]
    states, words = orc.rans_encode(tr["syms"], tr["freq"], lanes=tr["lanes"])
    assert states.tolist() == tr["states"]
    assert words.tolist() == tr["words"]
    st, back = orc.rans_decode(states, words, tr["syms"].size, tr["freq"], lanes=tr["lanes"])
    assert st == 0
    assert back.tolist() == tr["syms"].tolist()


def test_T2_table_from_counts(orc):
    """T2's table comes out of the normalisation of its own counts."""
    e = np.array([127, 127, 127, 126], np.uint8)
    f = orc.normalize(orc.histogram(e))
    assert f[126] == 1024 and f[127] == 3072 and int(f.sum()) == 4096


# ---------------------------------------------------------------- normalisation
@pytest.mark.parametrize("counts,expect", [
    ({0: 9997, 1: 1, 2: 1, 3: 1}, {0: 4093, 1: 1, 2: 1, 3: 1}),   # d = -1
    ({5: 1, 6: 1, 7: 1}, {5: 1366, 6: 1365, 7: 1365}),            # d = +1, tie -> lowest
    ({126: 1, 127: 3}, {126: 1024, 127: 3072}),                   # exact
    ({42: 7}, {42: 4096}),                                        # single symbol
    ({255: 123456789}, {255: 4096}),
    # d = -4 with a tie between two equal maxima: 10, 20, 10, 20 give up 1 each
    (dict([(10, 5000), (20, 5000)] + [(s, 1) for s in range(30, 40)]),
     dict([(10, 2043), (20, 2043)] + [(s, 1) for s in range(30, 40)])),
    # 255 rare symbols bumped to 1: the big one gives up 253 -> 4094 - 253
    (dict([(0, 1000000)] + [(s, 1) for s in range(1, 256)]),
     dict([(0, 3841)] + [(s, 1) for s in range(1, 256)])),
    # all 256 symbols equally likely
    ({s: 3 for s in range(256)}, {s: 16 for s in range(256)}),
])
def test_normalize_worked_examples(orc, counts, expect):
    f = orc.normalize(counts)
    want = np.zeros(256, np.uint16)
    for s, v in expect.items():
        want[s] = v
    assert f.tolist() == want.tolist()


def test_normalize_properties_random(orc):
    rng = np.random.default_rng(123)
    for trial in range(400):
        k = int(rng.integers(1, 257))
        present = rng.choice(256, size=k, replace=False)
        counts = np.zeros(256, np.uint64)
        scale = 10 ** int(rng.integers(0, 9))
        counts[present] = rng.integers(1, scale + 2, size=k).astype(np.uint64)
        if trial % 3 == 0:  # heavy skew
            counts[present[0]] *= np.uint64(10 ** 6)
        f = orc.normalize(counts).astype(np.int64)
        assert int(f.sum()) == 4096
        assert np.all(f[counts > 0] >= 1)
        assert np.all(f[counts == 0] == 0)
        # each frequency stays within its rounding window plus the correction:
        # |f - c*4096/n| < 1 + |d| where |d| <= number of present symbols
        n = float(counts.sum())
        ideal = counts.astype(np.float64) * 4096.0 / n
        assert np.all(np.abs(f - ideal)[counts > 0] <= 1 + k)


def test_normalize_empty(orc):
    assert orc.normalize(np.zeros(256, np.uint64)).tolist() == [0] * 256


# ---------------------------------------------------------------- brute force
def _tables(nsym_alpha, rng):
    """A few valid tables over symbols 0..nsym_alpha-1: extremes and random."""
    tabs = []
    a = nsym_alpha
    f = np.zeros(256, np.uint16)
    f[:a] = 1
    f[0] = 4096 - (a - 1)
    tabs.append(f.copy())
    f[:a] = 1
    f[a - 1] = 4096 - (a - 1)
    tabs.append(f.copy())
    for _ in range(2):
        cuts = np.sort(rng.choice(np.arange(1, 4096), size=a - 1, replace=False))
        parts = np.diff(np.concatenate([[0], cuts, [4096]]))
        g = np.zeros(256, np.uint16)
        g[:a] = parts
        tabs.append(g)
    return tabs


@pytest.mark.parametrize("lanes", [1, 32])
def test_brute_force_round_trip(orc, lanes):
    """Every sequence of length <= 6 over 2..4 symbols, several tables:
    decode(encode(x)) == x, every lane back at 2^16, every word read."""
    rng = np.random.default_rng(7)
    for alpha in (2, 3, 4):
        for tab in _tables(alpha, rng):
            for length in range(1, 7):
                for seq in itertools.product(range(alpha), repeat=length):
                    sym = np.array(seq, np.uint8)
                    states, words = orc.rans_encode(sym, tab, lanes=lanes)
                    assert np.all(states >= L)
                    st, back = orc.rans_decode(states, words, length, tab, lanes=lanes)
                    assert st == 0 and back.tolist() == list(seq)


def test_decoder_rejects_wrong_word_count(orc):
    tr = load_traces()["T3"]
    states, words = orc.rans_encode(tr["syms"], tr["freq"], lanes=32)
    st, _ = orc.rans_decode(states, words[:-1], tr["syms"].size, tr["freq"], lanes=32)
    assert st == 4
    st, _ = orc.rans_decode(states, np.concatenate([words, [7]]), tr["syms"].size, tr["freq"], lanes=32)
    assert st == 4
    bad = states.copy()
    bad[5] += 1
    st, _ = orc.rans_decode(bad, words, tr["syms"].size, tr["freq"], lanes=32)
    assert st == 4


# ---------------------------------------------------------------- accounting
def test_accounting_bound_and_entropy(orc):
    """|coded - ideal| <= exact slack for every chunk of workload 1, and the
    coded size is within 0.5% of the cross-entropy under the 12-bit table
    plus the fixed per-chunk overhead (128 state bytes, <= 15 pad bytes)."""
    import workloads
    bits = workloads.generate_tensor(1, 0)
    e, _ = orc.split_bf16(bits)
    f = orc.normalize(orc.histogram(e))
    cont = orc.encode(bits)
    n, dt, nc = orc.read_header(cont)
    off_len = 576 + 8 * (nc + 1)
    lens = cont[off_len: off_len + 4 * nc].view(np.uint32)
    for k in range(nc):
        sym = e[k * 65536:(k + 1) * 65536]
        coded, ideal, slack = orc.chunk_accounting(sym, f)
        assert abs(coded - ideal) <= slack + 1e-6
        assert slack < 5e-3 * ideal          # the bound itself is within 0.5%
        assert abs(coded - ideal) < 1e-4 * ideal
        assert lens[k] < 65536  # coded, not raw
        # coded bits = payload bits beyond the 32 x 16 state bits of L
        assert abs(8 * (int(lens[k]) - 128) + 32 * 16 - coded) < 32 * 17
        assert 8 * int(lens[k]) <= 1.005 * ideal + 8 * (128 + 15)


def test_exponent_statistics_sanity(orc):
    """N(0, 0.02) bf16: ~20 distinct exponents, ~2.5 bits/byte ("PTWM" How it
    works 2 reports ~20 values and ~2.6 bits/byte on trained weights)."""
    import workloads
    e, _ = orc.split_bf16(workloads.generate_tensor(1, 0))
    c = orc.histogram(e).astype(np.float64)
    p = c[c > 0] / c.sum()
    assert 15 <= (c > 0).sum() <= 30
    assert 2.3 < -(p * np.log2(p)).sum() < 2.8


# ---------------------------------------------------------------- planes
def test_split_bf16_worked(orc):
    bits = np.array([0xBF80, 0x3F81, 0x0001, 0xFFFF, 0x7F80], np.uint16)
    e, sm = orc.split_bf16(bits)
    assert e.tolist() == [127, 127, 0, 255, 255]
    assert sm.tolist() == [0x80, 0x01, 0x01, 0xFF, 0x00]


def test_split_fp32_worked(orc):
    bits = np.array([0x3F800000, 0xBF800000, 0x00000001, 0x7FC00000,
                     0x807FFFFF, 0x00000000, 0x00000000, 0x00000000,
                     0x80000000], np.uint32)
    e, sign, mant = orc.split_fp32(bits)
    assert e.tolist() == [127, 127, 0, 255, 0, 0, 0, 0, 0]
    assert sign.tolist() == [0b00010010, 0b00000001]
    assert mant[:15].tolist() == [0, 0, 0, 0, 0, 0, 1, 0, 0, 0, 0, 0x40, 0xFF, 0xFF, 0x7F]


def test_split_fp16_worked(orc):
    # fp16 S E5 M10; reordered E5 S M10; high byte coded, low byte raw
    bits = np.array([0x3C00, 0x8001, 0x7C00, 0xFC01, 0x7BFF, 0x3555, 0x0001, 0x8000], np.uint16)
    hi, lo = orc.split_fp16(bits)
    assert hi.tolist() == [0x78, 0x04, 0xF8, 0xFC, 0xF3, 0x69, 0x00, 0x04]
    assert lo.tolist() == [0x00, 0x01, 0x00, 0x01, 0xFF, 0x55, 0x01, 0x00]


def test_split_fp16_plane_structure(orc):
    # the coded byte is exponent << 3 | sign << 2 | top two mantissa bits
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 16, 4096, dtype=np.uint16)
    hi, lo = orc.split_fp16(bits)
    b = bits.astype(np.uint32)
    assert np.array_equal(hi >> 3, (b >> 10) & 0x1F)
    assert np.array_equal((hi >> 2) & 1, b >> 15)
    assert np.array_equal(hi & 3, (b >> 8) & 3)
    assert np.array_equal(lo, b & 0xFF)


def test_fp16_all_patterns_round_trip(orc):
    bits = np.arange(1 << 16, dtype=np.uint16)
    cont = orc.encode(bits, dtype=orc.FP16)
    assert orc.read_header(cont) == (1 << 16, orc.FP16, 1)
    assert np.array_equal(orc.decode(cont), bits)
    vals = (np.random.default_rng(4).standard_normal(5 * 65536 + 7) * 0.02).astype(np.float16)
    cont = orc.encode(vals)
    assert np.array_equal(orc.decode(cont), vals.view(np.uint16))
    assert cont.size < vals.nbytes          # the coded plane shrinks


def test_split_fp8e4m3_worked(orc):
    # fp8 e4m3 S E4 M3; reordered E4 | S M3; exponent nibble coded, low nibbles
    # raw, two per byte (even value in the low half)
    bits = np.array([0x38, 0xB8, 0x7E, 0x01, 0x80], np.uint8)
    e, nib = orc.split_fp8e4m3(bits)
    assert e.tolist() == [7, 7, 15, 0, 0]
    assert nib.tolist() == [0x80, 0x16, 0x08]


def test_split_fp8e4m3_plane_structure(orc):
    rng = np.random.default_rng(7)
    for n in (4096, 4097):
        bits = rng.integers(0, 256, n, dtype=np.uint8)
        e, nib = orc.split_fp8e4m3(bits)
        assert np.array_equal(e, (bits >> 3) & 0xF)
        lo = np.zeros(2 * nib.size, np.uint8)
        lo[0::2], lo[1::2] = nib & 0xF, nib >> 4
        assert np.array_equal(lo[:n], ((bits >> 4) & 8) | (bits & 7))
        assert n % 2 == 0 or lo[n] == 0          # the pad nibble is zero


def test_fp8e4m3_round_trips(orc):
    pats = np.arange(256, dtype=np.uint8)
    cont = orc.encode(pats)
    assert orc.read_header(cont) == (256, orc.FP8E4M3, 1)
    assert np.array_equal(orc.decode(cont), pats)
    rng = np.random.default_rng(8)
    # skewed: exponents around 7, with every pattern present
    vals = ((rng.integers(0, 2, 3 * 65536 + 7) << 7) | (np.clip(rng.normal(6, 1.2, 3 * 65536 + 7), 0, 15).astype(np.int64) << 3)
            | rng.integers(0, 8, 3 * 65536 + 7)).astype(np.uint8)
    vals[rng.choice(vals.size, 256, replace=False)] = pats
    cont = orc.encode(vals)
    assert np.array_equal(orc.decode(cont), vals)
    assert cont.size < vals.nbytes
    for n in (0, 1, 2, 3, 31, 33, 65535, 65537):
        v = vals[:n]
        c = orc.encode(v)
        assert np.array_equal(orc.decode(c), v)
        for k in range((n + 65535) // 65536):
            assert np.array_equal(orc.decode_chunk(c, k), v[k * 65536:(k + 1) * 65536])


def test_split_fp8e5m2_worked(orc):
    # fp8 e5m2 S E5 M2; reordered E5 S M2; high nibble (top four exponent bits)
    # coded, low nibble (lowest exponent bit, sign, mantissa) raw
    bits = np.array([0x3C, 0xBE, 0x7B, 0x01, 0x80], np.uint8)
    hi, nib = orc.split_fp8e5m2(bits)
    assert hi.tolist() == [7, 7, 15, 0, 0]
    # low nibbles 8, 0xE, 3, 1, 4 -> bytes 0xE8, 0x13, 0x04
    assert nib.tolist() == [0xE8, 0x13, 0x04]


def test_split_fp8e5m2_plane_structure(orc):
    rng = np.random.default_rng(17)
    for n in (4096, 4097):
        bits = rng.integers(0, 256, n, dtype=np.uint8)
        hi, nib = orc.split_fp8e5m2(bits)
        e5 = (bits >> 2) & 0x1F
        assert np.array_equal(hi, e5 >> 1)
        lo = ((e5 & 1) << 3) | ((bits >> 7) << 2) | (bits & 3)
        padded = np.zeros(2 * nib.size, np.uint8)
        padded[:n] = lo
        assert np.array_equal(nib, padded[0::2] | (padded[1::2] << 4))


def test_fp8e5m2_round_trips(orc):
    pats = np.arange(256, dtype=np.uint8)
    cont = orc.encode(pats, dtype=orc.FP8E5M2)
    assert orc.read_header(cont) == (256, orc.FP8E5M2, 1)
    assert np.array_equal(orc.decode(cont), pats)
    rng = np.random.default_rng(18)
    e = np.clip(rng.normal(13, 1.5, 3 * 65536 + 7), 0, 31).astype(np.int64)
    vals = ((rng.integers(0, 2, e.size) << 7) | (e << 2) | rng.integers(0, 4, e.size)).astype(np.uint8)
    vals[rng.choice(vals.size, 256, replace=False)] = pats
    cont = orc.encode(vals, dtype=orc.FP8E5M2)
    assert np.array_equal(orc.decode(cont), vals)
    assert cont.size < vals.nbytes
    for n in (0, 1, 2, 3, 33, 65537):
        v = vals[:n]
        c = orc.encode(v, dtype=orc.FP8E5M2)
        assert np.array_equal(orc.decode(c), v)
        for k in range((n + 65535) // 65536):
            assert np.array_equal(orc.decode_chunk(c, k), v[k * 65536:(k + 1) * 65536])


def test_split_bf16_highbyte_worked(orc):
    bits = np.array([0x3F80, 0xBF00, 0x0001, 0x7F80], np.uint16)
    hi, lo = orc.split_bf16_highbyte(bits)
    assert hi.tolist() == [0x3F, 0xBF, 0x00, 0x7F]
    assert lo.tolist() == [0x80, 0x00, 0x01, 0x80]


def test_bf16_highbyte_round_trips(orc):
    bits = np.arange(1 << 16, dtype=np.uint16)
    cont = orc.encode(bits, dtype=orc.BF16_HIGHBYTE)
    assert orc.read_header(cont) == (1 << 16, orc.BF16_HIGHBYTE, 1)
    assert np.array_equal(orc.decode(cont), bits)
    x = np.random.default_rng(19).standard_normal(3 * 65536 + 5).astype(np.float32) * np.float32(0.02)
    import workloads
    b = workloads.rne_bf16(x)
    cont = orc.encode(b, dtype=orc.BF16_HIGHBYTE)
    assert np.array_equal(orc.decode(cont), b)
    assert np.array_equal(orc.decode_chunk(cont, 3), b[3 * 65536:])
    # the coded plane is the high byte: same values, same table as counting
    # the high bytes directly
    hi, _ = orc.split_bf16_highbyte(b)
    assert np.array_equal(orc.histogram(hi), np.bincount(b >> 8, minlength=256))


# ---------------------------------------------------------------- containers
def test_golden_container_fp8e5m2_raw_chunk(orc):
    bits = np.array([0x3C, 0x3C, 0x3C, 0x38], np.uint8)
    want = load_container("container_fp8e5m2_n4_raw.txt")
    got = orc.encode(bits, dtype=orc.FP8E5M2)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()


def test_golden_container_bf16_highbyte_raw_chunk(orc):
    bits = np.array([0x3F80, 0x3F80, 0x3F80, 0x3F00], np.uint16)
    want = load_container("container_bf16_highbyte_n4_raw.txt")
    got = orc.encode(bits, dtype=orc.BF16_HIGHBYTE)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()


def test_golden_container_fp8e4m3_raw_chunk(orc):
    bits = np.array([0x38, 0x38, 0x38, 0x30], np.uint8)
    want = load_container("container_fp8e4m3_n4_raw.txt")
    got = orc.encode(bits)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()

def test_golden_container_fp16_raw_chunk(orc):
    bits = np.array([0x3C00, 0x3C00, 0x3C00, 0x3800], np.uint16)
    want = load_container("container_fp16_n4_raw.txt")
    got = orc.encode(bits, dtype=orc.FP16)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()


def test_golden_container_raw_chunk(orc):
    bits = np.array([0x3F80, 0x3F80, 0x3F80, 0x3F00], np.uint16)
    want = load_container("container_bf16_n4_raw.txt")
    got = orc.encode(bits)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()


def test_golden_container_single_symbol(orc):
    bits = np.full(200, 0x3F80, np.uint16)
    want = load_container("container_bf16_n200_single_symbol.txt")
    got = orc.encode(bits)
    assert got.size == want.size and np.array_equal(got, want)
    assert orc.decode(got).tolist() == bits.tolist()


def test_coded_payload_layout(orc):
    """A coded chunk's payload read as [32 x u32 states][w x u16 words]
    decodes with the rANS core to the chunk's exponents."""
    import workloads
    bits = workloads.generate_tensor(1, 0)[:100000]
    cont = orc.encode(bits)
    n, dt, nc = orc.read_header(cont)
    off_exp = int(cont[40:48].view(np.uint64)[0])
    choff = cont[576:576 + 8 * (nc + 1)].view(np.uint64)
    lens = cont[576 + 8 * (nc + 1): 576 + 8 * (nc + 1) + 4 * nc].view(np.uint32)
    f = cont[64:576].view(np.uint16)
    e, _ = orc.split_bf16(bits)
    for k in range(nc):
        nsym = min(65536, n - 65536 * k)
        p = off_exp + int(choff[k])
        assert lens[k] < nsym
        states = cont[p:p + 128].view(np.uint32)
        w = (int(lens[k]) - 128) // 2
        words = cont[p + 128:p + 128 + 2 * w].view(np.uint16)
        st, sym = orc.rans_decode(states, words, nsym, f)
        assert st == 0 and np.array_equal(sym, e[65536 * k:65536 * k + nsym])
        pad = cont[p + int(lens[k]): p + int(choff[k + 1] - choff[k])]
        assert not pad.any()


@pytest.mark.parametrize("fname,raw", [("container_bf16_n186_tie_raw.txt", True),
                                       ("container_bf16_n186_near_coded.txt", False)])
def test_golden_raw_fallback_boundary(orc, fname, raw):
    """The raw-fallback boundary ("PTWM" Configuration table,
    compression_threshold, read as: raw iff 128 + 2w >= nsym, ties raw): a
    chunk whose coded length equals nsym is stored raw, one 2 bytes shorter
    stays coded.  w comes from the pinned rANS core; the container bytes
    were laid out field by field, not by the oracle's encoder."""
    from _golden import load_fields
    e = np.array(load_fields(fname)["exponents"], np.uint8)
    bits = e.astype(np.uint16) << 7
    states, words = orc.rans_encode(e, orc.normalize(orc.histogram(e)))
    assert (128 + 2 * words.size == e.size) == raw
    assert (128 + 2 * words.size == e.size - 2) == (not raw)
    want = load_container(fname)
    got = orc.encode(bits)
    assert got.size == want.size and np.array_equal(got, want)
    chunk_len = int(got[592:596].view(np.uint32)[0])
    assert chunk_len == (e.size if raw else e.size - 2)
    assert orc.decode(got).tolist() == bits.tolist()
