"""The C-ABI library without a GPU: it loads, exports every entry point that
include/wc.h declares, sizes buffers like the oracle, parses headers like the
oracle, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wcm():
    from fp32_weight_compression_b200 import build, wc
    build.build()
    wc.load()
    return wc


def declared_entry_points():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"WC_API\s+[\w\s\*]*?\b(wc_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(wcm):
    names = declared_entry_points()
    assert len(names) >= 10
    lib = ctypes.CDLL(wcm.LIB_PATH)
    for nm in names:
        assert hasattr(lib, nm), nm
    assert set(wcm.EXPORTS) <= set(names)


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 65535, 65536, 65537, 10 ** 6, 123456789])
@pytest.mark.parametrize("dt", [1, 2])
def test_bound_matches_oracle(wcm, orc, n, dt):
    assert wcm.encode_bound(n, dt) == orc.encode_bound(n, dt)
    assert wcm.scratch_bytes(n, dt) >= 7424
    assert wcm.encode_bound(n, 5) == 0


def test_read_header_matches_oracle(wcm, orc):
    for n in (0, 1, 70000):
        for dt in ("bf16", "fp32"):
            x = (np.random.default_rng(n).standard_normal(n).astype(np.float32) * 0.02)
            bits = workloads.rne_bf16(x) if dt == "bf16" else x.view(np.uint32)
            cont = orc.encode(bits)
            assert wcm.read_header(cont) == orc.read_header(cont)
            assert wcm.read_header(cont[:64]) == orc.read_header(cont)


def test_read_header_rejects_corruption(wcm, orc):
    bits = workloads.generate_tensor(1, 0)[:100000]
    good = orc.encode(bits)
    for mutate in (lambda c: c.__setitem__(0, 0), lambda c: c.__setitem__(6, 9),
                   lambda c: c.__setitem__(7, 16), lambda c: c.__setitem__(64 + 2 * 3, 1),
                   lambda c: c.__setitem__(576 + 8, 7)):
        c = good.copy()
        mutate(c)
        with pytest.raises(wcm.WCError):
            wcm.read_header(c)


def test_bad_arguments_rejected_without_device(wcm):
    L = wcm.load()
    # misaligned input, output, scratch; too-small capacities; bad dtype
    cap = wcm.encode_bound(1000, 1)
    scr = wcm.scratch_bytes(1000, 1)
    ok_in, ok_out, ok_scr, ok_sz = 0x10000, 0x20000, 0x40000, 0x80000
    assert L.wc_encode(ok_in + 2, 1000, 1, ok_out, cap, ok_scr, scr, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_encode(ok_in, 1000, 1, ok_out + 8, cap, ok_scr, scr, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_encode(ok_in, 1000, 1, ok_out, cap, ok_scr + 16, scr, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_encode(ok_in, 1000, 1, ok_out, cap - 1, ok_scr, scr, ok_sz, None) == wcm.ERR_CAPACITY
    assert L.wc_encode(ok_in, 1000, 1, ok_out, cap, ok_scr, scr - 1, ok_sz, None) == wcm.ERR_CAPACITY
    assert L.wc_encode(ok_in, 1000, 7, ok_out, cap, ok_scr, scr, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_encode(None, 1000, 1, ok_out, cap, ok_scr, scr, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_decode(ok_in + 4, 1000, ok_out, 100, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_decode(ok_in, 1000, ok_out + 2, 100, ok_sz, None) == wcm.ERR_INVALID_ARG
    assert L.wc_decode(ok_in, 1000, ok_out, 100, None, None) == wcm.ERR_INVALID_ARG
    assert L.wc_decode_chunk(ok_in, 1000, 0, ok_out, 100, ok_sz + 2, None) == wcm.ERR_INVALID_ARG
    # block checksums: block size, alignment and null pointers
    assert L.wc_crc32_blocks(ok_in, 1000, 0, ok_out, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(ok_in, 1000, 4096, ok_out, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(ok_in, 1000, (1 << 30) + 8192, ok_out, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(ok_in + 8, 1000, 8192, ok_out, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(ok_in, 1000, 8192, ok_out + 2, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(None, 1000, 8192, ok_out, None) == wcm.ERR_INVALID_ARG
    assert L.wc_crc32_blocks(None, 0, 8192, None, None) == wcm.OK   # nothing to do
    assert wcm.status_string(4) == "WC_ERR_CORRUPT"


def test_product_path_has_no_oracle_dependency():
    """The library and its binding never reach the oracle or a CPU path."""
    pkg = os.path.join(ROOT, "fp32_weight_compression_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                for pat in ("import oracle", "from oracle", "liboracle", "wc_oracle",
                            "sys.path"):
                    assert pat not in text, (fn, pat)
