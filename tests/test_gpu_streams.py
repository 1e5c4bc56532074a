"""GPU: decode launches that overlap on several streams.  A decode launch's
blocks share out its work through a counter of its own (a slot of a
library-held array, zeroed on the launch's stream first); overlapping
launches must never share one, and a slot reused after the rotation has come
round must start from zero again."""
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


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def test_decodes_overlapping_on_four_streams(orc):
    from fp32_weight_compression_b200 import wc
    L = wc.load()
    sizes = [40 * C + 11, 33 * C, 17 * C + 5, 64 * C]
    bits = [workloads.rne_bf16(np.random.default_rng(70 + i).standard_normal(n).astype(np.float32)
                               * np.float32(0.02)) for i, n in enumerate(sizes)]
    conts = [wc.encode(_dev(b)) for b in bits]
    for b, c in zip(bits, conts):
        assert np.array_equal(c.cpu().numpy(), orc.encode(b))
    streams = [torch.cuda.Stream() for _ in sizes]
    outs = [[torch.empty(n, dtype=torch.bfloat16, device="cuda") for n in sizes] for _ in range(3)]
    status = torch.zeros(3, len(sizes), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for r in range(3):  # three rounds, no synchronisation between launches
        for i, (c, s) in enumerate(zip(conts, streams)):
            o = outs[r][i]
            assert L.wc_decode(c.data_ptr(), c.numel(), o.data_ptr(), 2 * o.numel(),
                               status[r, i:].data_ptr(), s.cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(status.abs().sum().item()) == 0
    for r in range(3):
        for b, o in zip(bits, outs[r]):
            assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), b)


def test_counter_slots_reused_after_the_rotation():
    from fp32_weight_compression_b200 import wc
    L = wc.load()
    b = workloads.generate_tensor(1, 0)[: 2 * C + 7].copy()
    c = wc.encode(_dev(b))
    out = torch.empty(b.size, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for k in range(4096 + 40):  # every slot once, then some again
        if k % 1024 == 1023 or k >= 4096:
            out.zero_()
        assert L.wc_decode(c.data_ptr(), c.numel(), out.data_ptr(), 2 * out.numel(), status.data_ptr(), s) == 0
        if k % 1024 == 1023 or k >= 4096:
            torch.cuda.synchronize()
            assert int(status.item()) == 0, k
            assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), b), k
