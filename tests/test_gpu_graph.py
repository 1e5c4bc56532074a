"""GPU: the batched encode and decode calls queue work only on the caller's
stream and never synchronise, so a CUDA graph can capture them and replay
the whole launch sequence.  A captured encode + decode of a mixed tensor set,
replayed on fresh input values written in place, gives the oracle's
containers and a bit-exact round trip each time."""
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
    return workloads.rne_bf16(x) if dt == "bf16" else x.view(np.uint32).copy()


def _to_dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a.view(np.int32)).view(torch.float32).cuda()


def test_captured_encode_decode_replays(orc):
    from fp32_weight_compression_b200 import wc
    sizes = [5 * C, 3 * C + 17, 100, 2 * C, C + 1]
    dts = ["bf16", "fp32", "bf16", "fp32", "bf16"]
    ins = [_to_dev(_bits(n, d, 40 + i)) for i, (n, d) in enumerate(zip(sizes, dts))]
    enc = wc.BatchEncoder([t.numel() for t in ins], [t.dtype for t in ins]).prepare(ins)
    conts_cap = [enc.out[o:o + c] for o, c in zip(enc.out_offsets, enc.caps)]
    outs = [torch.empty_like(t) for t in ins]
    dec = wc.BatchDecoder().prepare(conts_cap, outs)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):          # first calls outside capture (device set-up)
        enc.run()
        dec.run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        enc.run()
        dec.run()
    for rep in range(2):
        arrs = [_bits(n, d, 100 * rep + i) for i, (n, d) in enumerate(zip(sizes, dts))]
        for t, a in zip(ins, arrs):
            t.copy_(_to_dev(a))
        for o in outs:
            o.zero_()
        enc.out.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        dec.check()
        got = enc.containers()
        for a, c, o in zip(arrs, got, outs):
            assert np.array_equal(c.cpu().numpy(), orc.encode(a))
            view = torch.int16 if a.dtype == np.uint16 else torch.int32
            assert np.array_equal(o.view(view).cpu().numpy().view(a.dtype), a)
