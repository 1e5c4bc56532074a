"""Split12 serving format on the GPU (wc12_encode / wc12_decode through the C
ABI) against the numpy oracle (oracle/split12.py): containers byte-identical
for ragged sizes, exceptions in several chunks and steps, every bf16 pattern,
weight-like tensors; decoding of oracle-written containers; damaged
containers refused exactly when the oracle refuses them.  Collected after the
other GPU files."""
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
def s12():
    import split12
    return split12


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda")


def _check(s12, bits):
    from fp32_weight_compression_b200 import wc
    want = s12.encode(bits)
    cont = wc.split12_encode(_dev(bits))
    got = cont.cpu().numpy()
    assert got.size == want.size, (got.size, want.size)
    if not np.array_equal(got, want):
        diff = np.nonzero(got != want)[0]
        raise AssertionError(f"{diff.size} bytes differ, first at {diff[:8].tolist()}")
    back = wc.split12_decode(cont)
    assert np.array_equal(back.view(torch.int16).cpu().numpy().view(np.uint16), bits)


@pytest.mark.parametrize("n", [0, 1, 2, 15, 16, 17, 31, 4095, 4096, 4097, C - 1, C, C + 1,
                               3 * C + 4099])
def test_sizes(s12, n):
    _check(s12, workloads.generate_tensor(4, 1)[:n].copy())


def test_exceptions_across_chunks_and_steps(s12):
    b = workloads.generate_tensor(4, 1)[: 3 * C + 4099].copy()
    rng = np.random.default_rng(5)
    # rare high bytes spread over every chunk, in the first and last step of a
    # chunk, in neighbouring values and in the ragged tail
    pos = np.concatenate([[0, 1, 2, 15, 16, 4095, 4096, C - 1, C, 2 * C + 17, 3 * C + 4098],
                          rng.choice(b.size, 300, replace=False)])
    b[pos] = (rng.integers(0x40, 0x80, pos.size) << 8 | rng.integers(0, 256, pos.size)).astype(np.uint16)
    _check(s12, b)


def test_dense_exceptions_in_parts_of_a_chunk(s12):
    """Exception counts around the encoder's per-warp staging (256 entries
    for each eighth of a chunk, 8,192 values): exactly 256 in one eighth,
    257 in the next, a dense run across the boundary of two eighths, dense
    values in a ragged tail.  The other values take 16 high bytes only, so
    the codebook is those 16 and every other byte is an exception."""
    rng = np.random.default_rng(9)
    n = 2 * C + 3000
    book = np.array([0x3A, 0x3B, 0x3C, 0x3D, 0x3E, 0x3F, 0x40, 0x41,
                     0xBA, 0xBB, 0xBC, 0xBD, 0xBE, 0xBF, 0xC0, 0xC1], np.uint16)
    b = (book[rng.integers(0, 16, n)] << 8 | rng.integers(0, 256, n)).astype(np.uint16)
    others = np.setdiff1d(np.arange(256, dtype=np.uint16), book)
    rare = lambda k: (others[rng.integers(0, others.size, k)] << 8 | rng.integers(0, 256, k)).astype(np.uint16)
    E = C // 8
    for eighth, k in ((1, 256), (2, 257)):
        b[eighth * E + rng.choice(E, k, replace=False)] = rare(k)
    run = np.arange(C + 6 * E - 300, C + 6 * E + 400)          # across eighths 5 and 6 of chunk 1
    b[run] = rare(run.size)
    tail = np.arange(2 * C + 100, 2 * C + 2900)                 # the third chunk's 3,000 values
    b[tail] = rare(tail.size)
    hb = (b >> 8).astype(np.uint8)
    assert np.array_equal(s12.codebook(hb), book.astype(np.uint8))
    assert [int((~np.isin(hb[q * E:(q + 1) * E], book)).sum()) for q in (1, 2)] == [256, 257]
    assert s12.read_header(s12.encode(b))["ne"] == 256 + 257 + run.size + tail.size
    _check(s12, b)


def test_every_pattern_and_tiny_alphabets(s12):
    _check(s12, np.arange(1 << 16, dtype=np.uint16))                      # ne at its bound
    _check(s12, np.full(3 * C + 5, 0x3F80, np.uint16))                    # K = 1
    _check(s12, (np.arange(5 * C, dtype=np.uint16) % 16) << 8 | 0x55)     # K = 16, no exception


def test_weight_sets(s12):
    for cid, i in ((1, 0), (2, 0), (2, 196), (2, 200), (4, 4)):
        b = workloads.generate_tensor(cid, i)
        if b.size > 60_000_000:
            b = b[: 60_000_000 // C * C + 777]
        _check(s12, b)


def test_decodes_oracle_containers_and_refuses_damage(s12):
    from fp32_weight_compression_b200 import wc
    b = workloads.generate_tensor(4, 1)[: 2 * C + 999].copy()
    b[[3, C + 5, 2 * C + 998]] = 0x7001
    good = s12.encode(b)
    rng = np.random.default_rng(9)
    cases = [good]
    for _ in range(60):
        c = good.copy()
        for _ in range(int(rng.integers(1, 3))):
            region = int(rng.integers(0, 3))
            if region == 0:
                p = int(rng.integers(0, 96))                 # header, codebook, table start
            elif region == 1:
                p = int(rng.integers(0, c.size))            # anywhere
            else:
                p = int(rng.integers(c.size - 64, c.size))  # the exception lists
            c[p] ^= np.uint8(rng.integers(1, 256))
        cases.append(c)
    cases.append(good[:-16])
    for c in cases:
        try:
            want = s12.decode(c)
        except ValueError:
            want = None
        d = torch.zeros(c.size + 64, dtype=torch.uint8, device="cuda")
        d[: c.size] = torch.from_numpy(c)
        # room for a flipped n that still gives a valid, slightly longer
        # header; a guard region after it must stay untouched
        room = b.size + 1024
        out = torch.full((room + 2048,), 0x5A5A, dtype=torch.int16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert wc.load().wc12_decode(d.data_ptr(), c.size, out.data_ptr(), 2 * room,
                                     status.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
        torch.cuda.synchronize()
        st = int(status.item())
        assert bool((out[room:] == 0x5A5A).all().item())
        if want is None:
            assert st != 0
        else:
            assert st == 0
            assert np.array_equal(out[: want.size].cpu().numpy().view(np.uint16), want)


def test_batch_matches_single_calls_and_the_oracle(s12):
    """wc12_encode_batch / wc12_decode_batch: every container byte-identical
    to the oracle's, every value bit-exact, for a list of mixed sizes (empty,
    ragged, several chunks, exceptions) longer than one launch's 256 items."""
    from fp32_weight_compression_b200 import wc
    rng = np.random.default_rng(44)
    sizes = [0, 1, 17, C - 1, C, C + 1, 3 * C + 5] + [int(rng.integers(0, 3 * C)) for _ in range(290)]
    bits = []
    for i, n in enumerate(sizes):
        w = workloads.rne_bf16(rng.standard_normal(n).astype(np.float32) * np.float32(0.02))
        if n and i % 3 == 0:  # some exceptions
            m = rng.random(n) < 0.01
            w[m] = (rng.integers(0, 256, int(m.sum())) << 8).astype(np.uint16) | (w[m] & 0xFF)
        bits.append(w)
    conts = wc.split12_encode_batch([_dev(b) for b in bits])
    for b, c in zip(bits, conts):
        want = s12.encode(b)
        got = c.cpu().numpy()
        assert got.size == want.size and np.array_equal(got, want)
    outs = wc.split12_decode_batch(conts, [(b.size,) for b in bits])
    for b, o in zip(bits, outs):
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), b)


def test_batch_decode_refuses_a_wrong_count_and_damage(s12):
    from fp32_weight_compression_b200 import wc
    rng = np.random.default_rng(45)
    a = workloads.rne_bf16(rng.standard_normal(C + 9).astype(np.float32))
    b = workloads.rne_bf16(rng.standard_normal(2 * C).astype(np.float32))
    ca, cb = (torch.from_numpy(s12.encode(x)).to("cuda") for x in (a, b))
    with pytest.raises(wc.WCError) as ei:
        wc.split12_decode_batch([ca, cb], [(a.size,), (b.size - 1,)])  # not the tensor expected
    assert ei.value.code == wc.ERR_CORRUPT
    bad = ca.clone()
    bad[0] ^= 0xFF
    with pytest.raises(wc.WCError) as ei:
        wc.split12_decode_batch([bad, cb], [(a.size,), (b.size,)])
    assert ei.value.code == wc.ERR_CORRUPT
    outs = wc.split12_decode_batch([ca, cb], [(a.size,), (b.size,)])
    assert np.array_equal(outs[1].view(torch.int16).cpu().numpy().view(np.uint16), b)
