"""The coder's division by a symbol frequency, checked on the host.

The static rANS coding step ("SMEF -- blog companion code", pass4_rans.py;
"PTWM", How it works 2) needs
q = floor(x / f) for a renormalised state x < f 2^20.  When every frequency
of a tensor is at most 2048 the GPU coder computes it as
floor(x m / 2^k), k = 31 + ceil(log2 f), m = ceil(2^k / f) (a 32-bit
multiply-high and a shift); a tensor with a larger frequency uses a 64-bit
reciprocal instead.  These tests restate that rule in exact integer arithmetic
and check it against plain integer division where it is hardest (the largest
states, remainders f - 1), and show that the 2048 limit is needed."""
import numpy as np


def _narrow(f):
    c = (f - 1).bit_length()
    k = 31 + c
    return -(-(1 << k) // f), k


def _worst_states(f, span=4096):
    # q = 2^20 - j, r = f - 1: the error term x (m f - 2^k) / 2^k is largest
    # for the largest x, and a wrong floor shows first at r = f - 1
    j = np.arange(1, span + 1, dtype=np.uint64)
    return np.uint64(f) * (np.uint64(1 << 20) - j + np.uint64(1)) - np.uint64(1)


def test_multiplier_fits_32_bits():
    for f in range(2, 4097):
        m, _ = _narrow(f)
        assert m < 1 << 32, f


def test_exact_for_every_f_up_to_2048():
    rng = np.random.default_rng(0)
    for f in range(2, 2049):
        m, k = _narrow(f)
        x = np.concatenate([_worst_states(f),
                            rng.integers(0, f << 20, 2048, dtype=np.uint64),
                            np.arange(0, 4 * f, dtype=np.uint64)])
        q = (x * np.uint64(m)) >> np.uint64(k)          # x m < 2^31 2^32: no overflow
        assert np.array_equal(q, x // np.uint64(f)), f


def test_f_one_uses_all_ones_multiplier():
    # m = 2^32 - 1 without shift gives x - 1; the coder adds 4095 to cum to repay it
    x = np.arange(1, 1 << 20, 997, dtype=np.uint64)
    q = (x * np.uint64(0xFFFFFFFF)) >> np.uint64(32)
    assert np.array_equal(q, x - np.uint64(1))
    assert np.array_equal(x + q * np.uint64(4095) + np.uint64(4095), x * np.uint64(4096))


def test_limit_is_needed_above_2048():
    # some frequency above 2048 gets a wrong quotient from the narrow rule,
    # which is why such tables take the 64-bit path
    wrong = []
    for f in range(2049, 4096):
        m, k = _narrow(f)
        x = _worst_states(f, 64)
        if not np.array_equal((x * np.uint64(m)) >> np.uint64(k), x // np.uint64(f)):
            wrong.append(f)
    assert wrong and min(wrong) > 2048
