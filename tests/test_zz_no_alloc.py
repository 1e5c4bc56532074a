"""wc_encode_noalloc: encoding for callers that cannot allocate device memory
at the call site (a runtime that owns all device memory through a fixed
arena, a plug-in handed only its input and output buffers, a path that cannot
afford an allocator's implicit synchronisation).  Its scratch is a device
array the library holds; this file checks, through the C ABI, that its
containers are byte-identical to wc_encode's (which gets scratch from the
caller) and to the CPU oracle's, for bf16, fp32, fp16 and fp8 e4m3, on calls
in a row, and that inputs too large for the array are refused with
WC_ERR_CAPACITY before any work is queued.  Kept in a file of its own that pytest
collects after the parity files."""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu
MAX_VALUES = 248 * 65536  # the array serves 248 chunks


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp32_weight_compression_b200 import build
    build.build()


def _dev(bits, code=None):
    from fp32_weight_compression_b200 import wc
    if code == wc.FP16:
        return torch.from_numpy(bits.view(np.int16)).view(torch.float16).to("cuda")
    if code == wc.FP8E4M3:
        return torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).to("cuda")
    if bits.dtype == np.uint16:
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to("cuda")
    return torch.from_numpy(bits.view(np.int32)).view(torch.float32).to("cuda")


def _noalloc(lib, t, code):
    from fp32_weight_compression_b200 import wc
    n = t.numel()
    cap = wc.encode_bound(n, code)
    out = torch.full((cap,), 0xEE, dtype=torch.uint8, device="cuda")
    size = torch.zeros(1, dtype=torch.int64, device="cuda")
    rc = lib.wc_encode_noalloc(t.data_ptr(), n, code, out.data_ptr(), cap, size.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    torch.cuda.synchronize()
    return out[: int(size.item())]


def test_noalloc_matches_encode_on_calls_in_a_row(orc):
    from fp32_weight_compression_b200 import wc
    lib = wc.load()
    rng = np.random.default_rng(5)
    x32 = (rng.standard_normal(3 * 65536 + 4321).astype(np.float32) * np.float32(0.02))
    h16 = (rng.standard_normal(2 * 65536 + 77).astype(np.float32) * np.float32(0.05)).astype(np.float16)
    f8 = (rng.standard_normal(65536 + 999).astype(np.float32) * np.float32(4.0))
    f8 = torch.from_numpy(f8).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    cases = [
        (workloads.generate_tensor(1, 0), wc.BF16),                      # 16 chunks
        (x32.view(np.uint32).copy(), wc.FP32),                           # ragged fp32
        (h16.view(np.uint16).copy(), wc.FP16),                           # ragged fp16
        (f8, wc.FP8E4M3),                                                # ragged fp8 e4m3
        (workloads.adversarial_kind_tensor(0, 2), wc.BF16),              # raw fallback
        (workloads.generate_tensor(2, 196)[:MAX_VALUES].copy(), wc.BF16),  # largest accepted size
    ]
    for bits, code in cases:
        t = _dev(bits, code)
        ref = wc.encode(t)                 # existing entry point, caller scratch
        if code == wc.FP16:
            want = orc.encode(bits.view(np.float16))
        elif code == wc.FP8E4M3:
            want = orc.encode(bits)
        else:
            want = orc.encode(bits)
        for _ in range(2):                 # two calls in a row share the array
            got = _noalloc(lib, t, code)
            assert got.numel() == ref.numel()
            assert torch.equal(got, ref)
            assert np.array_equal(got.cpu().numpy(), want)   # and the oracle's container
        back = wc.decode(got, shape=t.shape, dtype=t.dtype)
        nbytes = {wc.BF16: torch.int16, wc.FP16: torch.int16, wc.FP32: torch.int32,
                  wc.FP8E4M3: torch.uint8}[code]
        assert torch.equal(back.view(nbytes), t.view(nbytes))


def test_noalloc_refuses_inputs_beyond_the_array():
    from fp32_weight_compression_b200 import wc
    lib = wc.load()
    assert wc.scratch_bytes(MAX_VALUES, wc.BF16) <= wc.NOALLOC_SCRATCH_BYTES
    assert wc.scratch_bytes(MAX_VALUES + 1, wc.BF16) > wc.NOALLOC_SCRATCH_BYTES
    # the size check comes before any use of the pointers
    for n in (MAX_VALUES + 1, 1 << 44, (1 << 44) + 1, (1 << 63)):
        for code in (wc.BF16, wc.FP32, wc.FP16, wc.FP8E4M3):
            rc = lib.wc_encode_noalloc(ctypes.c_void_p(0x1000), n, code, ctypes.c_void_p(0x2000),
                                       1 << 40, ctypes.c_void_p(0x3000), None)
            assert rc == wc.ERR_CAPACITY, (n, code)
    rc = lib.wc_encode_noalloc(ctypes.c_void_p(0x1000), 16, 99, ctypes.c_void_p(0x2000),
                               1 << 40, ctypes.c_void_p(0x3000), None)
    assert rc == wc.ERR_INVALID_ARG
