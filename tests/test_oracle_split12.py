"""Pins of the Split12 oracle (oracle/split12.py): a hand-worked container,
the 12-bits-a-value size, the codebook rule checked by brute force, round
trips over every bf16 pattern, and refusal of non-canonical containers."""
import numpy as np
import pytest

import workloads
from _golden import load_container

C = 65536


@pytest.fixture(scope="module")
def s12():
    import split12
    return split12


def _golden_bits():
    v = [0x3F80, 0x3F00] + [((i - 1) << 8) | (0xA0 + i) for i in range(2, 18)]
    return np.array(v, np.uint16)


def test_golden_container(s12):
    bits = _golden_bits()
    want = load_container("split12_n18_one_exception.txt")
    got = s12.encode(bits)
    assert got.size == want.size and np.array_equal(got, want)
    assert np.array_equal(s12.decode(got), bits)


def test_size_is_twelve_bits_a_value(s12):
    # no exceptions: header 64 + codebook 16 + offset table + n/2 + n bytes
    for n in (1, 2, 17, C, C + 1, 5 * C + 3):
        bits = np.full(n, 0x3C00, np.uint16) | np.arange(n, dtype=np.uint16) % 256
        cont = s12.encode(bits)
        nc = -(-n // C)
        r16 = lambda v: (v + 15) // 16 * 16
        assert cont.size == r16(r16(r16(80 + 8 * (nc + 1)) + (n + 1) // 2) + n)
        assert np.array_equal(s12.decode(cont), bits)
    big = s12.encode(np.full(64 * C, 0x3F80, np.uint16))
    assert abs(big.size / (2 * 64 * C) - 0.75) < 1e-4


def test_codebook_rule_by_brute_force(s12):
    rng = np.random.default_rng(12)
    for trial in range(200):
        nd = int(rng.integers(1, 40))
        alphabet = rng.choice(256, nd, replace=False)
        high = rng.choice(alphabet, int(rng.integers(1, 300))).astype(np.uint8)
        book = s12.codebook(high)
        counts = np.bincount(high, minlength=256)
        present = np.nonzero(counts)[0]
        assert book.size == min(16, present.size)
        assert np.all(np.diff(book.astype(int)) > 0)
        inside = set(book.tolist())
        for b in present:
            if b in inside:
                continue
            for a in inside:   # every member beats every outsider
                assert counts[a] > counts[b] or (counts[a] == counts[b] and a < b)


def test_round_trips(s12):
    every = np.arange(1 << 16, dtype=np.uint16)
    cont = s12.encode(every)
    h = s12.read_header(cont)
    assert h["k"] == 16 and h["ne"] == (256 - 16) * 256   # ties: bytes 0..15 win
    assert np.array_equal(s12.decode(cont), every)
    for n in (0, 1, 15, 16, 17, C - 1, C, C + 1):
        b = workloads.generate_tensor(4, 1)[:n]
        assert np.array_equal(s12.decode(s12.encode(b)), b)
    # exceptions in several chunks, the last one ragged
    b = workloads.generate_tensor(4, 1)[: 3 * C + 123].copy()
    b[[5, C + 7, 2 * C, 3 * C + 122]] = 0x0101
    cont = s12.encode(b)
    assert s12.read_header(cont)["ne"] >= 4
    assert np.array_equal(s12.decode(cont), b)


def test_ratio_on_weights(s12):
    # bf16 N(0, 0.02): a handful of exceptions, 12 bits a value plus a little
    b = workloads.generate_tensor(1, 0)
    cont = s12.encode(b)
    h = s12.read_header(cont)
    assert 0 < h["ne"] < b.size // 1000
    assert 0.75 < cont.size / b.nbytes < 0.7505


def test_structural_damage_refused(s12):
    good = s12.encode(_golden_bits())
    assert s12.canonical(good)
    cases = []
    c = good.copy(); c[144] = 30; cases.append(c)                     # exception past n
    c = good.copy(); c[0] = 0; cases.append(c)                        # magic
    c = good.copy(); c[88] = 2; cases.append(c)                       # exception count
    c = good.copy(); c[7] = 3; cases.append(c)                        # K = 3: index 15 out of range
    c = good.copy(); c[56] ^= 0x10; cases.append(c)                   # total
    for c in cases:
        with pytest.raises(ValueError):
            s12.decode(c)
    with pytest.raises(ValueError):
        s12.decode(good[:-1])                                         # cut short
    # two exceptions in one chunk must ascend
    b = np.arange(40, dtype=np.uint16) << 8 | 7
    cont = s12.encode(b)
    h = s12.read_header(cont)
    assert h["ne"] == 40 - 16
    bad = cont.copy()
    first_two = bad[h["off_exc"]:h["off_exc"] + 4].view("<u2").copy()
    bad[h["off_exc"]:h["off_exc"] + 4] = first_two[::-1].copy().view(np.uint8)
    with pytest.raises(ValueError):
        s12.decode(bad)


def test_non_canonical_detected(s12):
    good = s12.encode(_golden_bits())
    cases = []
    c = good.copy(); c[64:66] = [0x02, 0x01]; cases.append(c)        # codebook not ascending
    c = good.copy(); c[160] = 0x05; cases.append(c)                   # exception byte in the book
    c = good.copy(); c[104] = 0x1E; cases.append(c)                   # exception's index not 0
    # entry 14 (0x0F) replaced by 0x11: still ascending, but the decoded values
    # would then have 0x10 and 0x11 tied at one and 0x10 must win
    c = good.copy(); c[78] = 0x11; cases.append(c)
    for c in cases:
        s12.decode(c)                     # decodable, but not what encode writes
        assert not s12.canonical(c)
    # the valid container of other values is canonical
    c = good.copy(); c[79] = 0x3E
    assert s12.canonical(c)


def test_linear_worked_example(s12):
    # W = [[1, 2, -1], [0.5, 4, 3]] and x = [1, -2, 3] as bf16 bits;
    # x W^T = [1 - 4 - 3, 0.5 - 8 + 9] = [-6, 1.5], worked by hand
    w = np.array([0x3F80, 0x4000, 0xBF80, 0x3F00, 0x4080, 0x4040], np.uint16)
    x = np.array([[0x3F80, 0xC000, 0x4040]], np.uint16)
    y = s12.linear(x, s12.encode(w), 2)
    assert y.shape == (1, 2) and y.tolist() == [[-6.0, 1.5]]
    # two tokens, one with an exception in W (18 distinct high bytes)
    # 18 powers of four: exponents two apart, so 18 distinct high bytes
    vals = np.array([4.0 ** e for e in range(-9, 9)], np.float32)
    wb = (vals.view(np.uint32) >> 16).astype(np.uint16)               # exact in bf16
    xb = np.array([[0x3F80] * 18, [0x4000] * 9 + [0x0000] * 9], np.uint16)   # ones; twos then zeros
    y = s12.linear(xb, s12.encode(wb), 1)
    assert s12.read_header(s12.encode(wb))["ne"] == 2
    assert y[0, 0] == vals.astype(np.float64).sum()
    assert y[1, 0] == 2 * vals[:9].astype(np.float64).sum()


def test_random_inputs_round_trip_within_the_bound(s12):
    """Random alphabets and sizes: the oracle round-trips, its containers are
    canonical, and no container exceeds the size the library reserves
    (wc12_encode_bound: at most 15/16 of the values can be exceptions)."""
    from fp32_weight_compression_b200 import build, wc
    build.build()
    rng = np.random.default_rng(77)
    for trial in range(40):
        n = int(rng.choice([1, 2, 17, 255, 4097, C + 3, 2 * C + 1]))
        width = int(rng.integers(1, 257))
        highs = rng.choice(256, width, replace=False)
        p = rng.dirichlet(np.full(width, float(rng.choice([0.05, 1.0, 20.0]))))
        hi = rng.choice(highs, n, p=p).astype(np.uint16)
        bits = (hi << 8) | rng.integers(0, 256, n, dtype=np.uint16)
        cont = s12.encode(bits)
        assert np.array_equal(s12.decode(cont), bits)
        assert cont.size <= wc.split12_encode_bound(n)
        if trial % 8 == 0:
            assert s12.canonical(cont)
