"""The encoder's division by the symbol frequency, checked exhaustively on
the GPU (wc_check_coder_division, the same device function the encoder
runs): for every frequency f and every renormalised state x < f 2^20 the
coding step equals (x / f) 4096 + x % f + cum, in the 32-bit-multiplier
format (every f <= 2048) and in the 64-bit one (f up to 4095).  The coder's
step is the rANS encode step of "SMEF -- blog companion code" (pass4_rans.py)
with a 12-bit table."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp32_weight_compression_b200 import build
    build.build()


def test_narrow_format_exact_for_every_state():
    from fp32_weight_compression_b200 import wc
    assert wc.check_coder_division(False, 1, 2048) == (0, 0)


def test_wide_format_exact_for_every_state():
    from fp32_weight_compression_b200 import wc
    assert wc.check_coder_division(True, 1, 4095) == (0, 0)
