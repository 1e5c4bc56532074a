"""Host side of the windowed host<->device pipeline (wc_encode_host /
wc_decode_host) without a GPU: the window plan, the slot footprints, and the
argument checks that run before any CUDA call."""
import ctypes

import numpy as np
import pytest

import workloads


@pytest.fixture(scope="module")
def wcm():
    from fp32_weight_compression_b200 import build, wc
    build.build()
    wc.load()
    return wc


def r256(v):
    return (v + 255) // 256 * 256


def check_plan(fp, area, k, ends, target=0):
    slot = (area // k) // 256 * 256
    cap = target if 0 < target < slot else slot
    assert slot >= max(fp) + 256
    if k < 3:   # one more slot would not hold the largest item
        assert ((area // (k + 1)) // 256 * 256) < max(fp) + 256
    assert ends[-1] == len(fp) and all(a < b for a, b in zip(ends, ends[1:]))
    lo = 0
    for w, hi in enumerate(ends):
        used = 256 + sum(fp[lo:hi])
        assert used <= cap or hi == lo + 1     # an oversized item sits alone
        assert used <= slot
        if hi < len(fp):   # greedy: the next item would not have fitted
            assert used + fp[hi] > cap
        lo = hi


@pytest.mark.parametrize("seed", range(6))
def test_plan_is_greedy_and_fits(wcm, seed):
    rng = np.random.default_rng(seed)
    fp = [int(v) for v in rng.integers(1, 10 ** 6, int(rng.integers(1, 300)))]
    m = r256(max(fp) + 256)
    for area in (3 * m, 3 * m - 1, 2 * m + 300, m, 10 ** 8):
        for target in (0, 1, 4 * 10 ** 6, 10 ** 9):
            k, ends = wcm.host_plan(fp, area, target)
            check_plan(fp, area, k, ends, target)


def test_plan_slot_counts(wcm):
    # a slot must hold 1000 + 256 bytes, in whole 256-byte units: 1280
    assert wcm.host_plan([1000], 3 * 1280)[0] == 3
    assert wcm.host_plan([1000], 3 * 1280 - 1)[0] == 2
    assert wcm.host_plan([1000], 2 * 1280)[0] == 2
    assert wcm.host_plan([1000], 2 * 1280 - 1)[0] == 1
    assert wcm.host_plan([1000], 1280)[0] == 1
    with pytest.raises(wcm.WCError) as e:
        wcm.host_plan([1000], 1279)
    assert e.value.code == wcm.ERR_CAPACITY
    assert wcm.host_plan([], 10) == (0, [])
    with pytest.raises(wcm.WCError) as e:
        wcm.host_plan([5, 0], 10 ** 6)
    assert e.value.code == wcm.ERR_INVALID_ARG


@pytest.mark.parametrize("n", [0, 1, 65536, 65537, 10 ** 6])
@pytest.mark.parametrize("dt", [1, 2])
def test_footprints(wcm, n, dt):
    e = 2 if dt == 1 else 4
    assert wcm.host_encode_footprint(n, dt) == (r256(n * e) + r256(wcm.encode_bound(n, dt))
                                                + r256(wcm.scratch_bytes(n, dt)) + 8)
    assert wcm.host_decode_footprint(1000, n, dt) == r256(1000) + r256(n * e)
    assert wcm.host_encode_footprint(n, 6) == 0


def test_bad_arguments_rejected_before_device(wcm, orc):
    L = wcm.load()
    it = (wcm.HostEncodeItem * 1)()
    buf = np.zeros(4096, np.uint8)
    size = ctypes.c_uint64()
    it[0].h_in, it[0].n, it[0].dtype, it[0].reserved = buf.ctypes.data, 16, 1, 0
    it[0].h_out, it[0].h_out_cap, it[0].h_out_size = buf.ctypes.data, 4096, ctypes.addressof(size)
    assert L.wc_encode_host(it, 0, None, 0, 0, None, None, None) == wcm.OK
    assert L.wc_encode_host(None, 1, 256, 1 << 20, 0, None, None, None) == wcm.ERR_INVALID_ARG
    assert L.wc_encode_host(it, 1, 257, 1 << 20, 0, None, None, None) == wcm.ERR_INVALID_ARG
    it[0].dtype = 6
    assert L.wc_encode_host(it, 1, 256, 1 << 20, 0, None, None, None) == wcm.ERR_INVALID_ARG
    it[0].dtype, it[0].h_out_cap = 1, 10          # below wc_encode_bound
    assert L.wc_encode_host(it, 1, 256, 1 << 20, 0, None, None, None) == wcm.ERR_CAPACITY
    it[0].h_out_cap = 4096                         # workspace smaller than one slot
    assert L.wc_encode_host(it, 1, 256, 1024, 0, None, None, None) == wcm.ERR_CAPACITY

    st = ctypes.c_int32(7)
    di = (wcm.HostDecodeItem * 1)()
    bits = workloads.rne_bf16(np.ones(100, np.float32))
    cont = orc.encode(bits)
    out = np.zeros(100, np.uint16)
    di[0].h_cont, di[0].cont_bytes, di[0].h_out, di[0].out_cap = cont.ctypes.data, cont.size, out.ctypes.data, 200
    assert L.wc_decode_host(di, 1, 256, 1 << 20, 0, None, None, None, None) == wcm.ERR_INVALID_ARG
    di[0].out_cap = 199                            # too small for n = 100 bf16
    assert L.wc_decode_host(di, 1, 256, 1 << 20, 0, None, None, None, ctypes.byref(st)) == wcm.ERR_CAPACITY
    assert st.value == wcm.OK
    bad = cont.copy()
    bad[0] ^= 0xFF                                 # magic
    di[0].h_cont, di[0].out_cap = bad.ctypes.data, 200
    assert L.wc_decode_host(di, 1, 256, 1 << 20, 0, None, None, None, ctypes.byref(st)) == wcm.ERR_CORRUPT
