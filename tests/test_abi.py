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
            names += re.findall(r"WC_API\s+[\w\s\*]*?\b(wc(?:12)?_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(wcm):
    names = declared_entry_points()
    assert len(names) >= 10
    lib = ctypes.CDLL(wcm.LIB_PATH)
    for nm in names:
        assert hasattr(lib, nm), nm
    assert set(wcm.EXPORTS) <= set(names)


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 65535, 65536, 65537, 10 ** 6, 123456789])
@pytest.mark.parametrize("dt", [1, 2, 3, 4, 5])
def test_bound_matches_oracle(wcm, orc, n, dt):
    assert wcm.encode_bound(n, dt) == orc.encode_bound(n, dt)
    assert wcm.scratch_bytes(n, dt) >= 7424
    assert wcm.encode_bound(n, 6) == 0 and wcm.encode_bound(n, 0) == 0


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
    # the division self-check: ranges and the result pointer are checked first
    res = ctypes.c_void_p(0x10000)
    assert L.wc_check_coder_division(0, 1, 2049, res, None) == wcm.ERR_INVALID_ARG   # narrow <= 2048
    assert L.wc_check_coder_division(1, 1, 4096, res, None) == wcm.ERR_INVALID_ARG   # f <= 4095
    assert L.wc_check_coder_division(1, 0, 10, res, None) == wcm.ERR_INVALID_ARG     # f >= 1
    assert L.wc_check_coder_division(1, 9, 8, res, None) == wcm.ERR_INVALID_ARG      # empty range
    assert L.wc_check_coder_division(1, 1, 8, None, None) == wcm.ERR_INVALID_ARG
    assert L.wc_check_coder_division(1, 1, 8, ctypes.c_void_p(0x10004), None) == wcm.ERR_INVALID_ARG


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


def _masked_to_ranges(cont, ranges):
    keep = np.zeros_like(cont)
    for off, size in ranges:
        keep[off:off + size] = cont[off:off + size]
    return keep


@pytest.mark.parametrize("dt", ["bf16", "fp32", "fp16", "fp8"])
def test_chunk_ranges_hold_all_a_chunk_needs(wcm, orc, dt):
    """Every byte outside wc_chunk_ranges(k) zeroed: the oracle still decodes
    chunk k exactly, so the ranges hold everything that chunk needs."""
    rng = np.random.default_rng(31)
    n = 3 * 65536 + 100       # the last chunk (100 values) is always stored raw
    x = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    if dt == "bf16":
        bits = workloads.rne_bf16(x)
    elif dt == "fp32":
        bits = x.view(np.uint32).copy()
    elif dt == "fp16":
        bits = x.astype(np.float16)
    else:
        e = np.clip(rng.normal(6, 1.3, n), 0, 15).astype(np.int64)
        bits = ((rng.integers(0, 2, n) << 7) | (e << 3) | rng.integers(0, 8, n)).astype(np.uint8)
    # random bits in chunk 1 (stored raw except for fp8, whose 16-symbol
    # alphabet always codes below a byte per value)
    bits[65536:2 * 65536] = np.frombuffer(rng.bytes(65536 * bits.itemsize), bits.dtype)
    cont = orc.encode(bits)
    off_raw = int(cont[32:40].view(np.uint64)[0])
    raws = []
    for k in range(4):
        ranges = wcm.chunk_ranges(cont[:off_raw], k)
        assert ranges[0] == (0, off_raw)
        assert all(o % 16 == 0 or i > 0 for i, (o, _) in enumerate(ranges))
        assert sum(s for _, s in ranges) < cont.size
        part = _masked_to_ranges(cont, ranges)
        want = bits.reshape(-1)[k * 65536:(k + 1) * 65536]
        got = orc.decode_chunk(part, k)
        assert np.array_equal(got.view(np.uint8), want.view(np.uint8)), k
        # without any one of the data ranges the chunk no longer decodes
        for drop in range(1, len(ranges)):
            short = _masked_to_ranges(cont, ranges[:drop] + ranges[drop + 1:])
            try:
                bad = orc.decode_chunk(short, k)
                assert not np.array_equal(bad.view(np.uint8), want.view(np.uint8)), (k, drop)
            except orc.OracleError:
                pass
        n_, _, nc = orc.read_header(cont)
        lens = cont[576 + 8 * (nc + 1): 576 + 8 * (nc + 1) + 4 * nc].view(np.uint32)
        raws.append(int(lens[k]) == min(65536, n - k * 65536))
    assert raws[3] and not raws[0] and raws[1] == (dt != "fp8")


def test_chunk_ranges_rejects(wcm, orc):
    bits = workloads.rne_bf16(np.random.default_rng(2).standard_normal(70000).astype(np.float32))
    cont = orc.encode(bits)
    off_raw = int(cont[32:40].view(np.uint64)[0])
    with pytest.raises(wcm.WCError) as e:
        wcm.chunk_ranges(cont[:off_raw - 1], 0)               # prefix short of the tables
    assert e.value.code == wcm.ERR_CAPACITY
    with pytest.raises(wcm.WCError) as e:
        wcm.chunk_ranges(cont[:off_raw], 2)                   # only 2 chunks
    assert e.value.code == wcm.ERR_INVALID_ARG
    bad = cont[:off_raw].copy()
    bad[576 + 8] ^= 0x10                                      # chunk_off[1] off by 16
    with pytest.raises(wcm.WCError) as e:
        wcm.chunk_ranges(bad, 0)
    assert e.value.code == wcm.ERR_CORRUPT


@pytest.mark.parametrize("dt", ["bf16", "fp32", "fp16", "fp8"])
def test_header_fuzz_agrees_with_oracle(wcm, orc, dt):
    """Random byte flips in the header and tables: the library's host parser
    (wc_read_header) and the oracle accept and reject the same containers and
    read the same fields; where both accept, wc_chunk_ranges accepts too."""
    rng = np.random.default_rng(["bf16", "fp32", "fp16", "fp8"].index(dt) + 40)
    n = 3 * 65536 + 777
    x = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    bits = {"bf16": lambda: workloads.rne_bf16(x), "fp32": lambda: x.view(np.uint32).copy(),
            "fp16": lambda: x.astype(np.float16),
            "fp8": lambda: (np.clip(rng.normal(6, 1.3, n), 0, 15).astype(np.uint8) << 3)}[dt]()
    good = orc.encode(bits)
    off_raw = int(good[32:40].view(np.uint64)[0])
    both = 0
    for _ in range(600):
        c = good.copy()
        for _ in range(int(rng.integers(1, 3))):
            c[int(rng.integers(0, off_raw))] ^= np.uint8(rng.integers(1, 256))
        try:
            a = wcm.read_header(c)
        except wcm.WCError:
            a = None
        try:
            b = orc.read_header(c)
        except orc.OracleError:
            b = None
        assert a == b
        if a is not None:
            both += 1
            for k in range(a[2]):
                wcm.chunk_ranges(c[:off_raw], k)
    assert both < 600   # most flips must be caught


def test_split12_sizes_match_the_oracle_layout(wcm):
    import split12 as s12
    for n in (0, 1, 15, 16, 17, 65535, 65536, 65537, 5 * 65536 + 3):
        ne_max = n - (n + 15) // 16
        assert wcm.split12_encode_bound(n) == s12.layout(n, ne_max)["total"]
        assert wcm.split12_scratch_bytes(n) == 2560 + 1024 * (-(-n // 65536))
    # every bf16 pattern once: 240 of 256 high bytes missed, exactly the bound
    every = np.arange(1 << 16, dtype=np.uint16)
    assert s12.encode(every).size == wcm.split12_encode_bound(1 << 16)


def test_split12_bad_arguments_rejected_without_device(wcm):
    L = wcm.load()
    buf = (ctypes.c_uint8 * 4096)()
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    n = 100
    cap, scr = wcm.split12_encode_bound(n), wcm.split12_scratch_bytes(n)
    assert L.wc12_encode(base + 2, n, base, cap, base, scr, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode(base, n, base + 8, cap, base, scr, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode(base, n, base, cap, base + 4, scr, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode(base, n, base, cap, base, scr, base + 4, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode(None, n, base, cap, base, scr, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode(base, n, base, cap - 1, base, scr, base, None) == wcm.ERR_CAPACITY
    assert L.wc12_encode(base, n, base, cap, base, scr - 1, base, None) == wcm.ERR_CAPACITY
    assert L.wc12_decode(base + 4, 1000, base, 200, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_decode(base, 1000, base + 2, 200, base, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_decode(base, 1000, base, 200, None, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_decode(base, 1000, None, 200, base, None) == wcm.ERR_INVALID_ARG


def test_split12_linear_bad_arguments_rejected_without_device(wcm):
    L = wcm.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 255) // 256 * 256
    ok = dict(N=256, K=128, M=4)
    def call(w=b, N=ok["N"], K=ok["K"], x=b, M=ok["M"], y=b, st=b):
        return L.wc12_linear(w, 1 << 20, N, K, x, M, y, st, None)
    assert call(N=100) == wcm.ERR_INVALID_ARG          # N not a multiple of 128
    assert call(K=96) == wcm.ERR_INVALID_ARG           # K not a multiple of 64
    assert call(M=0) == wcm.ERR_INVALID_ARG
    assert call(w=b + 8) == wcm.ERR_INVALID_ARG        # container not 16-byte aligned
    assert call(x=b + 8) == wcm.ERR_INVALID_ARG
    assert call(y=b + 2) == wcm.ERR_INVALID_ARG
    assert call(w=None) == wcm.ERR_INVALID_ARG
    assert call(st=None) == wcm.ERR_INVALID_ARG
    assert L.wc12_linear(b, 95, 256, 128, b, 4, b, b, None) == wcm.ERR_INVALID_ARG   # no room for a header


def test_split12_batch_bad_arguments_rejected_without_device(wcm):
    L = wcm.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 255) // 256 * 256
    n = 100
    cap, scr = wcm.split12_encode_bound(n), wcm.split12_scratch_bytes(n)
    E = wcm.Split12EncodeItem
    def enc(**kw):
        f = dict(in_=b, n=n, out=b, out_cap=cap, scratch=b, scratch_cap=scr, out_size=b)
        f.update(kw)
        items = (E * 2)(E(**dict(f)), E(b, 1, b, wcm.split12_encode_bound(1), b, wcm.split12_scratch_bytes(1), b))
        return L.wc12_encode_batch(items, 2, None)
    assert enc(in_=b + 2) == wcm.ERR_INVALID_ARG
    assert enc(out=b + 8) == wcm.ERR_INVALID_ARG
    assert enc(out_size=b + 4) == wcm.ERR_INVALID_ARG
    assert enc(scratch=None) == wcm.ERR_INVALID_ARG
    assert enc(out_cap=cap - 1) == wcm.ERR_CAPACITY
    assert enc(scratch_cap=scr - 1) == wcm.ERR_CAPACITY
    assert L.wc12_encode_batch(None, 1, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_encode_batch(None, 0, None) == wcm.OK
    D = wcm.Split12DecodeItem
    items = (D * 1)(D(b + 4, 1000, b, 10))
    assert L.wc12_decode_batch(items, 1, b, None) == wcm.ERR_INVALID_ARG
    items = (D * 1)(D(b, 1000, b + 2, 10))
    assert L.wc12_decode_batch(items, 1, b, None) == wcm.ERR_INVALID_ARG
    items = (D * 1)(D(b, 1000, None, 10))
    assert L.wc12_decode_batch(items, 1, b, None) == wcm.ERR_INVALID_ARG
    items = (D * 1)(D(b, 1000, b, 10))
    assert L.wc12_decode_batch(items, 1, None, None) == wcm.ERR_INVALID_ARG


def test_split12_plan_size_and_bad_arguments(wcm):
    """wc12_plan_bytes from its layout; wc12_plan and wc12_linear_planned
    refuse bad arguments before touching a device."""
    L = wcm.load()
    for N, K, ne in ((128, 64, 0), (128, 64, 5), (4096, 14336, 22572), (256, 128, 1000)):
        nb = (N // 128) * (K // 64)
        off_ent = (32 + 4 * (nb + 1) + 15) // 16 * 16
        assert wcm.split12_plan_bytes(N, K, ne) == (off_ent + 4 * ne + 15) // 16 * 16
    buf = (ctypes.c_uint8 * 8192)()
    b = (ctypes.addressof(buf) + 255) // 256 * 256
    N, K = 128, 64
    pb = wcm.split12_plan_bytes(N, K, 3)
    big = 1 << 20
    assert L.wc12_plan(b + 8, big, N, K, 3, b, pb, b, None) == wcm.ERR_INVALID_ARG   # container alignment
    assert L.wc12_plan(b, big, N, K, 3, b + 8, pb, b, None) == wcm.ERR_INVALID_ARG   # plan alignment
    assert L.wc12_plan(b, big, 100, K, 3, b, pb, b, None) == wcm.ERR_INVALID_ARG     # N
    assert L.wc12_plan(b, big, N, 96, 3, b, pb, b, None) == wcm.ERR_INVALID_ARG      # K
    assert L.wc12_plan(b, big, N, K, N * K + 1, b, big, b, None) == wcm.ERR_INVALID_ARG  # ne > n
    assert L.wc12_plan(b, 100, N, K, 3, b, pb, b, None) == wcm.ERR_INVALID_ARG      # container too short
    assert L.wc12_plan(b, big, N, K, 3, b, pb - 16, b, None) == wcm.ERR_CAPACITY    # plan too short
    assert L.wc12_plan(b, big, N, K, 3, None, pb, b, None) == wcm.ERR_INVALID_ARG
    assert L.wc12_plan(b, big, N, K, 3, b, pb, None, None) == wcm.ERR_INVALID_ARG
    def planned(plan=b, plan_bytes=pb, N=256, K=128, M=4):
        return L.wc12_linear_planned(b, big, plan, plan_bytes, N, K, b, M, b, b, None)
    assert planned(plan=None) == wcm.ERR_INVALID_ARG
    assert planned(plan=b + 8) == wcm.ERR_INVALID_ARG
    assert planned(plan_bytes=40) == wcm.ERR_INVALID_ARG        # below the header and starts
    assert planned(N=100) == wcm.ERR_INVALID_ARG
    assert planned(M=0) == wcm.ERR_INVALID_ARG


def test_split12_read_header_matches_the_oracle(wcm):
    import split12 as s12
    rng = np.random.default_rng(12)
    for n in (0, 1, 17, 65537):
        bits = (rng.integers(0, 40, n).astype(np.uint16) << 8) | rng.integers(0, 256, n).astype(np.uint16)
        cont = s12.encode(bits)
        h = s12.read_header(cont)
        assert wcm.split12_read_header(cont) == (h["n"], h["ne"], h["k"])
        # the library's header checks refuse what the oracle's refuse
        for _ in range(200):
            c = cont.copy()
            c[int(rng.integers(0, 64))] ^= np.uint8(rng.integers(1, 256))
            try:
                s12.read_header(c)
                ok = True
            except ValueError:
                ok = False
            try:
                wcm.split12_read_header(c)
                got = True
            except wcm.WCError:
                got = False
            assert got == ok
        with pytest.raises(wcm.WCError):
            wcm.split12_read_header(cont[:-1])


def test_headers_are_plain_c_and_link(wcm, tmp_path):
    """The public headers compile as C99 (-pedantic, no warnings), every
    declared entry point links from libwc.so, and size queries answer from a
    C program as they do through the binding."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    names = declared_entry_points()
    src = ['#include <stdio.h>', '#include "wc.h"', '#include "wc_split12.h"', '#include "wc_diag.h"',
           'typedef void (*fn_t)(void);',
           'int main(void) {', '  const fn_t fns[] = {']
    src += [f'    (fn_t)&{n},' for n in names]
    src += ['  };', '  (void)fns;',
            '  printf("%llu %llu %llu\\n", (unsigned long long)wc_encode_bound(1000, WC_FP32),',
            '         (unsigned long long)wc12_encode_bound(1000), (unsigned long long)wc_scratch_bytes(1000, WC_BF16));',
            '  return 0;', '}']
    c = tmp_path / "abi.c"
    c.write_text("\n".join(src) + "\n")
    pkg = os.path.join(ROOT, "fp32_weight_compression_b200")
    exe = tmp_path / "abi"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-Wno-cast-function-type", "-I", os.path.join(ROOT, "include"), str(c), "-L", pkg,
                        "-lwc", f"-Wl,-rpath,{pkg}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert [int(v) for v in out] == [wcm.encode_bound(1000, 2), wcm.split12_encode_bound(1000),
                                     wcm.scratch_bytes(1000, 1)]
