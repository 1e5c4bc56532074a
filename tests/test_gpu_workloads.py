"""Full-size parity on the five workloads, in the launch configuration the
benchmark times (one batched encode and one batched decode over the whole
tensor set): every container is byte-identical to the CPU oracle's (compared
by SHA-256; the oracle runs in spawn-started worker processes), and every
tensor round-trips bit-exactly, on all five workloads (workload 4: 225
tensors, 15.0 GB)."""
import hashlib
import multiprocessing as mp

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


def _pool():
    return mp.get_context("spawn").Pool(min(16, workloads.default_workers()))


def _one_to_device(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to("cuda")
    return torch.from_numpy(a.view(np.int32)).view(torch.float32).to("cuda")


def _to_device(arrs):
    return [_one_to_device(a) for a in arrs]


def _generate_on_device(pool, cid, idx):
    """Draw the tensors in the worker pool and move each to the device as it
    arrives (host memory holds a few tensors at a time)."""
    from workload_oracle import gen_tensor
    out = {}
    for i, a in pool.imap_unordered(gen_tensor, [(cid, i) for i in idx]):
        out[i] = _one_to_device(a)
        del a
    return [out[i] for i in idx]


def _encode_decode(ts):
    from fp32_weight_compression_b200 import wc
    enc = wc.BatchEncoder([t.numel() for t in ts], [t.dtype for t in ts])
    enc.prepare(ts).run()
    conts_cap = [enc.out[o:o + c] for o, c in zip(enc.out_offsets, enc.caps)]
    outs = [torch.empty_like(t) for t in ts]
    dec = wc.BatchDecoder().prepare(conts_cap, outs).run()
    torch.cuda.synchronize()
    dec.check()
    sizes = enc.sizes.cpu().tolist()
    return enc, sizes, outs


def _bitwise_equal(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def _digest(t):
    return hashlib.sha256(t.cpu().numpy().tobytes()).hexdigest()


@pytest.mark.parametrize("cid", [2, 3, 5])
def test_workload_full_parity(cid):
    from workload_oracle import oracle_digest
    specs = workloads.tensor_specs(cid)
    idx = list(range(len(specs)))
    with _pool() as pool:
        digests = pool.map_async(oracle_digest, [(cid, i) for i in idx])
        ts = _generate_on_device(pool, cid, idx)
        want = {i: (n, h) for i, n, h in digests.get()}
    enc, sizes, outs = _encode_decode(ts)
    conts = enc.containers(sizes)
    for i in idx:
        n, h = want[i]
        assert sizes[i] == n, (specs[i].name, sizes[i], n)
        assert _digest(conts[i]) == h, specs[i].name
        assert _bitwise_equal(outs[i], ts[i]), specs[i].name



def test_workload4_full_parity():
    """All 225 tensors (15.0 GB): every container byte-identical to the
    oracle's (SHA-256 of each, computed in the worker that drew the tensor),
    every tensor round-trips bit-exactly, and random access on the
    525M-value embedding decodes chunks in place."""
    from fp32_weight_compression_b200 import wc
    from workload_oracle import gen_tensor_and_digest
    cid = 4
    specs = workloads.tensor_specs(cid)
    idx = list(range(len(specs)))
    emb = len(specs) - 1
    ts, want = {}, {}
    with _pool() as pool:
        for i, a, n, h in pool.imap_unordered(gen_tensor_and_digest, [(cid, i) for i in idx]):
            ts[i] = _one_to_device(a)
            want[i] = (n, h)
            del a
    ts = [ts[i] for i in idx]
    enc, sizes, outs = _encode_decode(ts)
    conts = enc.containers(sizes)
    for i in idx:
        n, h = want[i]
        assert sizes[i] == n, (specs[i].name, sizes[i], n)
        assert _digest(conts[i]) == h, specs[i].name
        assert _bitwise_equal(outs[i], ts[i]), specs[i].name
    ce = conts[emb]
    assert int(ce[20:24].cpu().numpy().view(np.uint32)[0]) == 8016
    for k in (0, 4007, 8015):
        v = wc.decode_chunk(ce, k)
        assert _bitwise_equal(v, ts[emb].reshape(-1)[k * C:(k + 1) * C]), k


def test_workload5_kinds_standalone_parity(orc):
    """Each adversarial kind as its own tensor (1 and 3 chunks): kind (b)
    then has a single-symbol table, kind (a) is all raw."""
    from fp32_weight_compression_b200 import wc
    for kind in range(4):
        for nch in (1, 3):
            bits = workloads.adversarial_kind_tensor(kind, nch)
            t = _to_device([bits])[0]
            cont = wc.encode(t)
            assert np.array_equal(cont.cpu().numpy(), orc.encode(bits)), (kind, nch)
            back = wc.decode(cont, shape=t.shape, dtype=t.dtype)
            assert _bitwise_equal(back, t)
