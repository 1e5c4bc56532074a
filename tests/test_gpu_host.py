"""GPU: the windowed host<->device pipeline (wc_encode_host / wc_decode_host)
produces exactly the oracle's containers from host tensors and decodes host
containers bit-exactly, with one, two and three workspace slots and many
windows; a corrupted container is reported through the status word."""
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


def _bits(n, dt, seed):
    x = np.random.default_rng(seed).standard_normal(n).astype(np.float32) * np.float32(0.02)
    if dt == "fp16":
        return x.astype(np.float16)
    if dt == "fp8":
        e = np.clip(np.random.default_rng(seed).normal(6, 1.3, n), 0, 15).astype(np.int64)
        return ((e << 3) | (np.arange(n) % 8) | ((np.arange(n) % 3 == 0) << 7)).astype(np.uint8)
    return workloads.rne_bf16(x) if dt == "bf16" else x.view(np.uint32).copy()


def _host(bits, pin=True):
    if bits.dtype == np.uint16:
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    elif bits.dtype == np.float16:
        t = torch.from_numpy(bits.view(np.int16)).view(torch.float16)
    elif bits.dtype == np.uint8:
        t = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn)
    else:
        t = torch.from_numpy(bits.view(np.int32)).view(torch.float32)
    return t.pin_memory() if pin else t.clone()


def _set():
    sizes = [0, 1, 100, C - 3, C, C + 5, 3 * C + 17, 5 * C, 17, 2 * C + 1]
    kinds = ["fp32", "bf16", "fp16", "fp8"]
    return [_bits(n, kinds[i % 4], 500 + i) for i, n in enumerate(sizes)]


@pytest.mark.parametrize("window", [1, 1 << 20, 0])    # one item per window .. one slot per window
@pytest.mark.parametrize("slots", [3, 2, 1])
def test_host_round_trip_matches_oracle(orc, slots, window):
    from fp32_weight_compression_b200 import wc
    arrs = _set()
    ts = [_host(a) for a in arrs]
    code = {np.dtype(np.uint16): 1, np.dtype(np.uint32): 2, np.dtype(np.float16): 3,
            np.dtype(np.uint8): 4}
    big = max(wc.host_encode_footprint(a.size, code[a.dtype]) for a in arrs)
    slot = (big + 256 + 255) // 256 * 256
    work = 256 * ((4 * len(arrs) + 255) // 256) + slots * slot   # status words + slots
    codec = wc.HostCodec(work, window_bytes=window)
    conts = codec.encode(ts)
    for a, c in zip(arrs, conts):
        assert np.array_equal(c.numpy(), orc.encode(a))
    outs = codec.decode(conts)
    for a, o in zip(arrs, outs):
        got = o.view({4: torch.int32, 2: torch.int16, 1: torch.uint8}[a.dtype.itemsize]).numpy()
        assert np.array_equal(got.view(a.dtype), a)


def test_host_pageable_buffers_and_reuse():
    from fp32_weight_compression_b200 import wc
    arrs = _set()
    ts = [_host(a, pin=False) for a in arrs]
    codec = wc.HostCodec(64 << 20)
    outs, sizes = codec.encode_buffers(ts, pin=False)
    first = [c.clone() for c in codec.encode(ts, outs, sizes)]
    again = codec.encode(ts, outs, sizes)
    assert all(torch.equal(a, b) for a, b in zip(first, again))
    dev = wc.encode_batch([t.cuda() for t in ts])
    assert all(torch.equal(a, d.cpu()) for a, d in zip(first, dev))


def test_host_decode_reports_corruption(orc):
    from fp32_weight_compression_b200 import wc
    bits = _bits(4 * C, "bf16", 9)
    cont = torch.from_numpy(orc.encode(bits)).pin_memory()
    hdr = cont[:64].numpy()
    off_exp = int(hdr[40:48].view(np.uint64)[0])
    bad = cont.clone()
    bad[off_exp + 5] ^= 0x5A                       # a state byte of chunk 0
    codec = wc.HostCodec(64 << 20)
    with pytest.raises(wc.WCError) as e:
        codec.decode([cont, bad])
    assert e.value.code == wc.ERR_CORRUPT
    out = codec.decode([cont])[0]
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), bits)
