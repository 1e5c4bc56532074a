// k_encode.cu -- encoder stage 2: plane split + rANS coding per chunk, and the
// exclusive scan of chunk sizes into the container's offset table.
//
// A block of 8 warps codes 16 consecutive chunks of one tensor, two per warp
// (one rANS state per lane per chunk, symbol i in lane i mod 32).  Two full
// chunks (any dtype) are coded in lock-step, so every lane carries two
// independent state chains; other chunks are coded one at a time.  A warp
// walks a chunk backwards in groups of 512 values (16 steps): each lane loads
// its 16 consecutive values, writes their raw planes straight into the
// container's raw section (bf16: the sign+mantissa byte; fp16: the low byte;
// fp32: sign bits and 3 little-endian mantissa bytes -- "PTWM" How it works
// 1-2, "SMEF" pass3_streams.py), and parks their coded bytes (the exponent;
// for fp16 the reordered high byte) in shared memory, where step t reads byte
// 32 t + lane.  Coding a symbol s with frequency f from
// state x (12-bit table, L = 2^16, 16-bit words):
//   if x >= f 2^20: emit x & 0xFFFF, x >>= 16;   x = (x / f) 4096 + x % f + cum_s
// with x / f computed exactly by a multiply-high and a shift when every f of
// the tensor is at most 2048 (the usual case), else by a 64-bit reciprocal in
// two 32-bit halves (see publish_table); the coder is compiled for both and
// each block takes the form its tensor's table was written in.  The lanes
// that emit at a step form one block of the word stream, in ascending lane
// order, placed with __ballot_sync / __popc prefix offsets; blocks are laid
// down back to front, so the decoder (which runs the steps forwards) reads
// them in order.  A chunk stops coding as soon as 128 + 2w >= nsym: it will be
// stored raw ("PTWM" Configuration table, compression_threshold).
//
// The last warp to finish a tensor scans the tensor's chunk lengths into
// chunk_off[] (16-byte rounded) and chunk_len[] and completes the header.
#include "wc_block.cuh"
#include "wc_coder.cuh"
#include "wc_format.cuh"
#include "wc_hist.cuh"
#include "wc_planes.cuh"

namespace wc {

constexpr int kCoderThreads = kCoderWarps * 32;

// Per-block shared state of the coder, at namespace scope so that helper
// functions reach it as shared memory (not through generic pointers).
__shared__ uint4 s_tab[256];
__shared__ uint32_t s_bias[256];
__shared__ __align__(16) uint8_t s_ebuf[kCoderWarps][2][kGroupValues];
__shared__ uint32_t s_len[kCoderWarps][2];

// ---------------------------------------------------------------------------
// 16 consecutive 2-byte values (bf16 or fp16, 8 words) of one lane: their
// coded bytes and raw bytes (wc_planes.cuh).
struct V16x16 {
  uint4 a, b;
};

template <int DT>
__device__ __forceinline__ uint4 codes16(const V16x16 &v) {
  return make_uint4(code4<DT>(v.a.x, v.a.y), code4<DT>(v.a.z, v.a.w), code4<DT>(v.b.x, v.b.y),
                    code4<DT>(v.b.z, v.b.w));
}
template <int DT>
__device__ __forceinline__ uint4 raws16(const V16x16 &v) {
  return make_uint4(raw4<DT>(v.a.x, v.a.y), raw4<DT>(v.a.z, v.a.w), raw4<DT>(v.b.x, v.b.y),
                    raw4<DT>(v.b.z, v.b.w));
}

// fp32: exponent byte = byte 3 of (u << 1)
__device__ __forceinline__ uint32_t exp4_fp32(uint4 u) {
  const uint32_t p01 = __byte_perm(u.x << 1, u.y << 1, 0x0073);
  const uint32_t p23 = __byte_perm(u.z << 1, u.w << 1, 0x0073);
  return __byte_perm(p01, p23, 0x5410);
}
// 4 mantissas (23 bits) as 12 little-endian bytes
__device__ __forceinline__ uint3 mant4_fp32(uint4 u) {
  const uint32_t m0 = u.x & 0x7FFFFFu, m1 = u.y & 0x7FFFFFu, m2 = u.z & 0x7FFFFFu, m3 = u.w & 0x7FFFFFu;
  return make_uint3(m0 | (m1 << 24), (m1 >> 8) | (m2 << 16), (m2 >> 16) | (m3 << 8));
}
__device__ __forceinline__ uint32_t sign4_fp32(uint4 u) {
  return (u.x >> 31) | ((u.y >> 31) << 1) | ((u.z >> 31) << 2) | ((u.w >> 31) << 3);
}

// Raw planes and exponents of one value (ragged tails only).
template <int DT>
__device__ __forceinline__ uint32_t one_value(const uint8_t *in, uint64_t vg, uint8_t *out, const Layout &L) {
  static_assert(!is_fp8(DT), "fp8 raw nibbles are written a byte (two values) at a time");
  if (DT != WC_FP32) {
    const uint32_t b = reinterpret_cast<const uint16_t *>(in)[vg];
    out[L.off_raw + vg] = uint8_t(raw_byte<DT>(b));
    return code_byte<DT>(b);
  } else {
    const uint32_t u = reinterpret_cast<const uint32_t *>(in)[vg];
    const uint32_t m = u & 0x7FFFFFu;
    uint8_t *md = out + L.off_mant + 3 * vg;
    md[0] = uint8_t(m);
    md[1] = uint8_t(m >> 8);
    md[2] = uint8_t(m >> 16);
    return (u >> 23) & 0xFFu;
  }
}

// One coding step of one lane.
template <bool W>
__device__ __forceinline__ void cstep(uint32_t &x, uint32_t &tail, uint16_t *win16, const uint4 *tab,
                                      const uint32_t *bias, uint32_t s, uint32_t lt) {
  const uint4 te = tab[s];
  const uint32_t bi = W ? bias[s] : 0u;
  const bool emit = x > te.y;
  const uint32_t m = __ballot_sync(0xffffffffu, emit);
  tail -= __popc(m);
  if (emit) win16[tail + __popc(m & lt)] = uint16_t(x);
  x = emit ? (x >> 16) : x;
  x = advance<W>(x, te, bi);
}

// One coding step of two chains, interleaved operation by operation.
template <bool W>
__device__ __forceinline__ void cstep2(uint32_t &xA, uint32_t &tA, uint16_t *wA, uint32_t sA,
                                       uint32_t &xB, uint32_t &tB, uint16_t *wB, uint32_t sB,
                                       const uint4 *tab, const uint32_t *bias, uint32_t lt) {
  const uint4 eA = tab[sA], eB = tab[sB];
  const uint32_t bA = W ? bias[sA] : 0u, bB = W ? bias[sB] : 0u;
  const bool pA = xA > eA.y, pB = xB > eB.y;
  const uint32_t mA = __ballot_sync(0xffffffffu, pA);
  const uint32_t mB = __ballot_sync(0xffffffffu, pB);
  tA -= __popc(mA);
  tB -= __popc(mB);
  if (pA) wA[tA + __popc(mA & lt)] = uint16_t(xA);
  if (pB) wB[tB + __popc(mB & lt)] = uint16_t(xB);
  xA = pA ? (xA >> 16) : xA;
  xB = pB ? (xB >> 16) : xB;
  xA = advance<W>(xA, eA, bA);
  xB = advance<W>(xB, eB, bB);
}

// A step that may hold lanes past nsym.
template <bool W>
__device__ __forceinline__ void cstep_checked(uint32_t &x, uint32_t &tail, uint16_t *win16,
                                              const uint4 *tab, const uint32_t *bias, uint32_t s,
                                              bool valid, uint32_t lt) {
  const uint4 te = tab[s];
  const uint32_t bi = W ? bias[s] : 0u;
  const bool emit = valid && x > te.y;
  const uint32_t m = __ballot_sync(0xffffffffu, emit);
  const uint32_t k = __popc(m);
  if (emit) {
    win16[tail - k + __popc(m & lt)] = uint16_t(x);
    x >>= 16;
  }
  tail -= k;
  if (valid) x = advance<W>(x, te, bi);
}

struct CoderOut {
  uint32_t *lens;  // the warp's two chunk lengths (shared memory)
  uint64_t k0;     // the warp's first chunk
  uint8_t *win0;   // window of chunk 0 of the tensor
};

// A chunk's stored length: 128 + 2w if that is smaller than nsym, else nsym
// (raw).  A coded chunk's final states go to the front of its window.
__device__ __forceinline__ void finish_chunk(const CoderOut &co, uint64_t k, uint32_t nsym, uint32_t x,
                                             uint32_t tail, bool bail, int lane) {
  const uint32_t w = kWinWords - tail;
  const bool raw = bail || (kStateBytes + 2 * w >= nsym);
  const uint32_t len = raw ? nsym : kStateBytes + 2 * w;
  if (!raw) reinterpret_cast<uint32_t *>(co.win0 + k * kWin)[lane] = x;
  if (lane == 0) co.lens[k - co.k0] = len;
}

// Two full 2-byte-value chunks (bf16 or fp16) kA, kA + 1 in lock-step.
template <int DT, bool W>
__device__ __forceinline__ void code_pair16(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
                               const uint32_t *bias, uint8_t *ebA, uint8_t *ebB, const CoderOut &co) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const uint64_t vgA = kA * kChunk, vgB = vgA + kChunk;
  const uint16_t *in16 = reinterpret_cast<const uint16_t *>(it.in);
  uint16_t *wA = reinterpret_cast<uint16_t *>(co.win0 + kA * kWin);
  uint16_t *wB = reinterpret_cast<uint16_t *>(co.win0 + (kA + 1) * kWin);
  uint32_t xA = kStateLow, xB = kStateLow, tA = kWinWords, tB = kWinWords;
  bool bailA = false, bailB = false;
  constexpr int NG = int(kChunk / kGroupValues);

  V16x16 cA, cB, nA, nB;
  {
    const uint64_t o = uint64_t(NG - 1) * kGroupValues + 16 * lane;
    cA.a = ld_nc_v4(in16 + vgA + o); cA.b = ld_nc_v4(in16 + vgA + o + 8);
    cB.a = ld_nc_v4(in16 + vgB + o); cB.b = ld_nc_v4(in16 + vgB + o + 8);
  }
  for (int G = NG - 1; G >= 0; --G) {
    const uint64_t o = uint64_t(G) * kGroupValues + 16 * lane;
    st_cs_v4(it.out + L.off_raw + vgA + o, raws16<DT>(cA));
    st_cs_v4(it.out + L.off_raw + vgB + o, raws16<DT>(cB));
    *reinterpret_cast<uint4 *>(ebA + 16 * lane) = codes16<DT>(cA);
    *reinterpret_cast<uint4 *>(ebB + 16 * lane) = codes16<DT>(cB);
    if (G > 0) {
      const uint64_t on = o - kGroupValues;
      nA.a = ld_nc_v4(in16 + vgA + on); nA.b = ld_nc_v4(in16 + vgA + on + 8);
      nB.a = ld_nc_v4(in16 + vgB + on); nB.b = ld_nc_v4(in16 + vgB + on + 8);
    }
    __syncwarp();
    if (!bailA && !bailB) {
#pragma unroll
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep2<W>(xA, tA, wA, ebA[32 * t + lane], xB, tB, wB, ebB[32 * t + lane], tab, bias, lt);
    } else if (!bailA) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xA, tA, wA, tab, bias, ebA[32 * t + lane], lt);
    } else if (!bailB) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xB, tB, wB, tab, bias, ebB[32 * t + lane], lt);
    }
    if (kStateBytes + 2 * (kWinWords - tA) >= kChunk) bailA = true;
    if (kStateBytes + 2 * (kWinWords - tB) >= kChunk) bailB = true;
    __syncwarp();
    cA = nA;
    cB = nB;
  }
  finish_chunk(co, kA, kChunk, xA, tA, bailA, lane);
  finish_chunk(co, kA + 1, kChunk, xB, tB, bailB, lane);
}

// 16 consecutive fp32 values of one lane.
struct Fp32x16 {
  uint4 a, b, c, d;
};

__device__ __forceinline__ void load_fp32x16(const uint32_t *p, Fp32x16 &v) {
  v.a = ld_nc_v4(p);
  v.b = ld_nc_v4(p + 4);
  v.c = ld_nc_v4(p + 8);
  v.d = ld_nc_v4(p + 12);
}

// Raw planes of 16 fp32 values (value vg is a multiple of 16) into the
// container; their exponent bytes into eb.
__device__ __forceinline__ void split_fp32x16(const Fp32x16 &v, uint8_t *out, const Layout &L,
                                              uint64_t vg, uint8_t *eb) {
  const uint32_t sb = sign4_fp32(v.a) | (sign4_fp32(v.b) << 4) | (sign4_fp32(v.c) << 8) |
                      (sign4_fp32(v.d) << 12);
  *reinterpret_cast<uint16_t *>(out + L.off_raw + vg / 8) = uint16_t(sb);
  const uint3 m0 = mant4_fp32(v.a), m1 = mant4_fp32(v.b), m2 = mant4_fp32(v.c), m3 = mant4_fp32(v.d);
  uint8_t *md = out + L.off_mant + 3 * vg;
  st_cs_v4(md, make_uint4(m0.x, m0.y, m0.z, m1.x));
  st_cs_v4(md + 16, make_uint4(m1.y, m1.z, m2.x, m2.y));
  st_cs_v4(md + 32, make_uint4(m2.z, m3.x, m3.y, m3.z));
  *reinterpret_cast<uint4 *>(eb) = make_uint4(exp4_fp32(v.a), exp4_fp32(v.b), exp4_fp32(v.c), exp4_fp32(v.d));
}

// Two full fp32 chunks kA, kA + 1 in lock-step (as code_pair16; the next
// group's values are loaded into the registers the current group's split
// has just freed).
template <bool W>
__device__ __forceinline__ void code_pair_fp32(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
                               const uint32_t *bias, uint8_t *ebA, uint8_t *ebB, const CoderOut &co) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const uint64_t vgA = kA * kChunk, vgB = vgA + kChunk;
  const uint32_t *in32 = reinterpret_cast<const uint32_t *>(it.in);
  uint16_t *wA = reinterpret_cast<uint16_t *>(co.win0 + kA * kWin);
  uint16_t *wB = reinterpret_cast<uint16_t *>(co.win0 + (kA + 1) * kWin);
  uint32_t xA = kStateLow, xB = kStateLow, tA = kWinWords, tB = kWinWords;
  bool bailA = false, bailB = false;
  constexpr int NG = int(kChunk / kGroupValues);

  Fp32x16 vA, vB;
  {
    const uint64_t o = uint64_t(NG - 1) * kGroupValues + 16 * lane;
    load_fp32x16(in32 + vgA + o, vA);
    load_fp32x16(in32 + vgB + o, vB);
  }
  for (int G = NG - 1; G >= 0; --G) {
    const uint64_t o = uint64_t(G) * kGroupValues + 16 * lane;
    split_fp32x16(vA, it.out, L, vgA + o, ebA + 16 * lane);
    split_fp32x16(vB, it.out, L, vgB + o, ebB + 16 * lane);
    if (G > 0) {
      load_fp32x16(in32 + vgA + o - kGroupValues, vA);
      load_fp32x16(in32 + vgB + o - kGroupValues, vB);
    }
    __syncwarp();
    if (!bailA && !bailB) {
#pragma unroll
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep2<W>(xA, tA, wA, ebA[32 * t + lane], xB, tB, wB, ebB[32 * t + lane], tab, bias, lt);
    } else if (!bailA) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xA, tA, wA, tab, bias, ebA[32 * t + lane], lt);
    } else if (!bailB) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xB, tB, wB, tab, bias, ebB[32 * t + lane], lt);
    }
    if (kStateBytes + 2 * (kWinWords - tA) >= kChunk) bailA = true;
    if (kStateBytes + 2 * (kWinWords - tB) >= kChunk) bailB = true;
    __syncwarp();
  }
  finish_chunk(co, kA, kChunk, xA, tA, bailA, lane);
  finish_chunk(co, kA + 1, kChunk, xB, tB, bailB, lane);
}

// Two full fp8 e4m3 chunks kA, kA + 1 in lock-step (as code_pair16: 16
// values are one 16-byte load; their low nibbles are 8 bytes of the plane).
template <int DT, bool W>
__device__ __forceinline__ void code_pair8(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
                           const uint32_t *bias, uint8_t *ebA, uint8_t *ebB, const CoderOut &co) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const uint64_t vgA = kA * kChunk, vgB = vgA + kChunk;
  uint16_t *wA = reinterpret_cast<uint16_t *>(co.win0 + kA * kWin);
  uint16_t *wB = reinterpret_cast<uint16_t *>(co.win0 + (kA + 1) * kWin);
  uint32_t xA = kStateLow, xB = kStateLow, tA = kWinWords, tB = kWinWords;
  bool bailA = false, bailB = false;
  constexpr int NG = int(kChunk / kGroupValues);

  uint4 cA, cB, nA, nB;
  {
    const uint64_t o = uint64_t(NG - 1) * kGroupValues + 16 * lane;
    cA = ld_nc_v4(it.in + vgA + o);
    cB = ld_nc_v4(it.in + vgB + o);
  }
  for (int G = NG - 1; G >= 0; --G) {
    const uint64_t o = uint64_t(G) * kGroupValues + 16 * lane;
    st_cs_v2(it.out + L.off_raw + (vgA + o) / 2,
             make_uint2(fp8_pack8<DT>(cA.x, cA.y), fp8_pack8<DT>(cA.z, cA.w)));
    st_cs_v2(it.out + L.off_raw + (vgB + o) / 2,
             make_uint2(fp8_pack8<DT>(cB.x, cB.y), fp8_pack8<DT>(cB.z, cB.w)));
    *reinterpret_cast<uint4 *>(ebA + 16 * lane) =
        make_uint4(fp8_code4(cA.x), fp8_code4(cA.y), fp8_code4(cA.z), fp8_code4(cA.w));
    *reinterpret_cast<uint4 *>(ebB + 16 * lane) =
        make_uint4(fp8_code4(cB.x), fp8_code4(cB.y), fp8_code4(cB.z), fp8_code4(cB.w));
    if (G > 0) {
      nA = ld_nc_v4(it.in + vgA + o - kGroupValues);
      nB = ld_nc_v4(it.in + vgB + o - kGroupValues);
    }
    __syncwarp();
    if (!bailA && !bailB) {
#pragma unroll
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep2<W>(xA, tA, wA, ebA[32 * t + lane], xB, tB, wB, ebB[32 * t + lane], tab, bias, lt);
    } else if (!bailA) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xA, tA, wA, tab, bias, ebA[32 * t + lane], lt);
    } else if (!bailB) {
#pragma unroll 4
      for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
        cstep<W>(xB, tB, wB, tab, bias, ebB[32 * t + lane], lt);
    }
    if (kStateBytes + 2 * (kWinWords - tA) >= kChunk) bailA = true;
    if (kStateBytes + 2 * (kWinWords - tB) >= kChunk) bailB = true;
    __syncwarp();
    cA = nA;
    cB = nB;
  }
  finish_chunk(co, kA, kChunk, xA, tA, bailA, lane);
  finish_chunk(co, kA + 1, kChunk, xB, tB, bailB, lane);
}

// Any single chunk (either dtype, possibly ragged).
template <int DT, bool W>
__device__ __noinline__ void code_one(const EncItem &it, const Layout &L, uint64_t k, int slot,
                                      const CoderOut &co) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint4 *tab = s_tab;
  const uint32_t *bias = s_bias;
  uint8_t *eb = s_ebuf[warp][slot];
  const uint32_t lt = lanemask_lt();
  const uint32_t nsym = chunk_nsym(it.n, k);
  const int ngroups = int((nsym + kGroupValues - 1) / kGroupValues);
  const uint64_t vg0 = k * kChunk;
  uint16_t *win16 = reinterpret_cast<uint16_t *>(co.win0 + k * kWin);
  uint32_t x = kStateLow, tail = kWinWords;
  bool bail = false;

  for (int G = ngroups - 1; G >= 0; --G) {
    const uint32_t gb = uint32_t(G) * kGroupValues;
    const uint32_t vl = gb + 16 * lane;  // lane's first value in the chunk
    const uint64_t vg = vg0 + vl;
    if (vl + 16 <= nsym) {
      uint4 e;
      if constexpr (is_fp8(DT)) {
        const uint4 v = ld_nc_v4(it.in + vg);
        st_cs_v2(it.out + L.off_raw + vg / 2, make_uint2(fp8_pack8<DT>(v.x, v.y), fp8_pack8<DT>(v.z, v.w)));
        e = make_uint4(fp8_code4(v.x), fp8_code4(v.y), fp8_code4(v.z), fp8_code4(v.w));
      } else if constexpr (DT != WC_FP32) {
        const uint16_t *p = reinterpret_cast<const uint16_t *>(it.in) + vg;
        V16x16 v;
        v.a = ld_nc_v4(p);
        v.b = ld_nc_v4(p + 8);
        st_cs_v4(it.out + L.off_raw + vg, raws16<DT>(v));
        e = codes16<DT>(v);
      } else {
        const uint32_t *p = reinterpret_cast<const uint32_t *>(it.in) + vg;
        const uint4 u0 = ld_nc_v4(p), u1 = ld_nc_v4(p + 4), u2 = ld_nc_v4(p + 8), u3 = ld_nc_v4(p + 12);
        e = make_uint4(exp4_fp32(u0), exp4_fp32(u1), exp4_fp32(u2), exp4_fp32(u3));
        const uint32_t sb = sign4_fp32(u0) | (sign4_fp32(u1) << 4) | (sign4_fp32(u2) << 8) |
                            (sign4_fp32(u3) << 12);
        *reinterpret_cast<uint16_t *>(it.out + L.off_raw + vg / 8) = uint16_t(sb);
        const uint3 m0 = mant4_fp32(u0), m1 = mant4_fp32(u1), m2 = mant4_fp32(u2), m3 = mant4_fp32(u3);
        uint8_t *md = it.out + L.off_mant + 3 * vg;
        st_cs_v4(md, make_uint4(m0.x, m0.y, m0.z, m1.x));
        st_cs_v4(md + 16, make_uint4(m1.y, m1.z, m2.x, m2.y));
        st_cs_v4(md + 32, make_uint4(m2.z, m3.x, m3.y, m3.z));
      }
      *reinterpret_cast<uint4 *>(eb + 16 * lane) = e;
    } else if constexpr (is_fp8(DT)) {
      // ragged tail: a byte of the nibble plane holds two values (the second
      // nibble is zero past nsym); coded bytes past nsym are zero
      for (uint32_t q = 0; q < 8; q++) {
        const bool v0 = vl + 2 * q < nsym, v1 = vl + 2 * q + 1 < nsym;
        const uint32_t b0 = v0 ? it.in[vg + 2 * q] : 0u, b1 = v1 ? it.in[vg + 2 * q + 1] : 0u;
        eb[16 * lane + 2 * q] = uint8_t(v0 ? fp8_code(b0) : 0u);
        eb[16 * lane + 2 * q + 1] = uint8_t(v1 ? fp8_code(b1) : 0u);
        if (v0) it.out[L.off_raw + (vg + 2 * q) / 2] = uint8_t(fp8_nibble<DT>(b0) | (v1 ? fp8_nibble<DT>(b1) << 4 : 0u));
      }
    } else {
      // ragged tail: value by value; exponent bytes past nsym are zero
      for (uint32_t j = 0; j < 16; j++) {
        uint32_t e = 0;
        if (vl + j < nsym) e = one_value<DT>(it.in, vg + j, it.out, L);
        eb[16 * lane + j] = uint8_t(e);
      }
      if (DT == WC_FP32) {
        for (uint32_t bsel = 0; bsel < 2; bsel++) {
          if (vl + 8 * bsel >= nsym) break;
          uint32_t byte = 0;
          for (uint32_t j = 0; j < 8 && vl + 8 * bsel + j < nsym; j++)
            byte |= (reinterpret_cast<const uint32_t *>(it.in)[vg + 8 * bsel + j] >> 31) << j;
          it.out[L.off_raw + (vg + 8 * bsel) / 8] = uint8_t(byte);
        }
      }
    }
    __syncwarp();
    if (!bail) {
      if (gb + kGroupValues <= nsym) {
#pragma unroll 4
        for (int t = int(kStepsPerGroup) - 1; t >= 0; --t)
          cstep<W>(x, tail, win16, tab, bias, eb[32 * t + lane], lt);
      } else {
        const int steps = int((nsym - gb + 31) / 32);
        for (int t = steps - 1; t >= 0; --t)
          cstep_checked<W>(x, tail, win16, tab, bias, eb[32 * t + lane], gb + 32 * t + lane < nsym, lt);
      }
      if (kStateBytes + 2 * (kWinWords - tail) >= nsym) bail = true;
    }
    __syncwarp();
  }
  finish_chunk(co, k, nsym, x, tail, bail, lane);
}

// The warp's two chunks kA and (if hasB) kA + 1.
template <int DT, bool W>
__device__ __forceinline__ void code_warp(const EncItem &it, const Layout &L, uint64_t kA, bool hasB,
                                          int warp, const CoderOut &co) {
  if (hasB && chunk_nsym(it.n, kA + 1) == kChunk) {
    if (DT == WC_FP32) code_pair_fp32<W>(it, L, kA, s_tab, s_bias, s_ebuf[warp][0], s_ebuf[warp][1], co);
    else if (is_fp8(DT)) code_pair8<DT, W>(it, L, kA, s_tab, s_bias, s_ebuf[warp][0], s_ebuf[warp][1], co);
    else code_pair16<DT, W>(it, L, kA, s_tab, s_bias, s_ebuf[warp][0], s_ebuf[warp][1], co);
  } else {
    code_one<DT, W>(it, L, kA, 0, co);
    if (hasB) code_one<DT, W>(it, L, kA + 1, 1, co);
  }
}

// ---------------------------------------------------------------------------
// Header fields, padding and scratch counters (one block per tensor).
__global__ void __launch_bounds__(256) k_prep(const __grid_constant__ EncParams p) {
  const EncItem &it = p.items[blockIdx.x];
  const int tid = threadIdx.x;
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);
  uint8_t *out = it.out;

  uint64_t *hist = reinterpret_cast<uint64_t *>(it.scratch + kScrHist);
  uint32_t *ctr = reinterpret_cast<uint32_t *>(it.scratch + kScrCtr);
  uint64_t *stat = reinterpret_cast<uint64_t *>(it.scratch + kScrStat);
  hist[tid] = 0;
  if (tid < 4) ctr[tid] = 0;
  for (uint64_t k = tid; k < L.nc; k += 256) stat[k] = 0;

  // table: all zero until the last histogram tile writes it (n = 0 keeps it)
  reinterpret_cast<uint16_t *>(out + kFreqOffset)[tid] = 0;

  if (tid == 0) {
    uint32_t *h32 = reinterpret_cast<uint32_t *>(out);
    uint64_t *h64 = reinterpret_cast<uint64_t *>(out);
    h32[0] = 0x315A4357u;  // "WCZ1"
    h32[1] = kVersion | (uint32_t(dtype) << 16) | (kLanes << 24);
    h64[1] = it.n;
    h32[4] = kChunk;
    h32[5] = uint32_t(L.nc);
    h32[6] = kProbBits;  // u16 12, u16 0
    h32[7] = 0;
    h64[4] = L.off_raw;
    h64[5] = L.off_exp;
    if (it.n == 0) {
      h64[6] = 0;
      h64[7] = L.off_exp;
      *reinterpret_cast<uint64_t *>(out + L.off_chunk_off) = 0;
      *it.out_size = L.off_exp;
    }
  }
  // zero padding: after the chunk-length table, and after each raw plane
  if (tid < 16) {
    uint64_t a = L.off_chunk_len + 4 * L.nc + tid;
    if (a < L.off_raw) out[a] = 0;
    if (dtype != WC_FP32) {
      const uint64_t raw_bytes = is_fp8(dtype) ? (it.n + 1) / 2 : it.n;
      uint64_t b = L.off_raw + raw_bytes + tid;
      if (b < L.off_exp) out[b] = 0;
    } else {
      uint64_t b = L.off_raw + (it.n + 7) / 8 + tid;
      if (b < L.off_mant) out[b] = 0;
      uint64_t c = L.off_mant + 3 * it.n + tid;
      if (c < L.off_exp) out[c] = 0;
    }
  }
}

// ---------------------------------------------------------------------------
// k_hist: one block (512 threads) per tile of 4 chunks counts the tile's coded
// bytes and adds them to the tensor's histogram; the tensor's last tile turns
// the counts into the table.  The whole GPU reads the input at memory speed.
//
// k_encode: persistent coding.  Blocks take coding tasks (16 chunks of one
// tensor, two per warp) in order from a counter, so every task that a task
// waits for was taken earlier by a running block.  A warp that has coded its
// chunks places them with a decoupled look-back over the tensor's per-chunk
// words (stat): it publishes each chunk's padded length, reads its
// predecessors' words (32 at a time) until one holds an inclusive prefix,
// publishes its own inclusive prefix, writes the offset-table entries and
// copies the payload from its window (or the raw exponent bytes from the
// input) to the final place, zero-padded to 16 bytes.  The last chunk of a
// tensor completes the header and the size.  A predecessor waits only for
// its own coding, so the waits end; each is bounded all the same (kWaitNs),
// and a tensor whose wait ran out gets size 0.

constexpr int kHistThreads = 512;

__shared__ uint32_t s_task;
__shared__ uint32_t s_flag;

// bytes [mis, mis + 16) of the 32 bytes a:b (mis even, 0..14)
__device__ __forceinline__ uint4 extract16(uint4 a, uint4 b, uint32_t mis) {
  const uint32_t sh = (mis & 3u) * 8u;
  uint32_t r0, r1, r2, r3, r4;
  switch (mis >> 2) {
    case 0: r0 = a.x; r1 = a.y; r2 = a.z; r3 = a.w; r4 = b.x; break;
    case 1: r0 = a.y; r1 = a.z; r2 = a.w; r3 = b.x; r4 = b.y; break;
    case 2: r0 = a.z; r1 = a.w; r2 = b.x; r3 = b.y; r4 = b.z; break;
    default: r0 = a.w; r1 = b.x; r2 = b.y; r3 = b.z; r4 = b.w; break;
  }
  return make_uint4(__funnelshift_r(r0, r1, sh), __funnelshift_r(r1, r2, sh),
                    __funnelshift_r(r2, r3, sh), __funnelshift_r(r3, r4, sh));
}

__device__ __forceinline__ uint32_t keep_bytes(uint32_t v, int keep) {
  if (keep >= 4) return v;
  if (keep <= 0) return 0;
  return v & ((1u << (8 * keep)) - 1u);
}
__device__ __forceinline__ uint4 keep16(uint4 o, int keep) {
  if (keep >= 16) return o;
  return make_uint4(keep_bytes(o.x, keep), keep_bytes(o.y, keep - 4), keep_bytes(o.z, keep - 8),
                    keep_bytes(o.w, keep - 12));
}

// A coded chunk's payload: the 32 states (front of the window) and the w
// words (the window's last 2w bytes, 2-byte aligned; realigned here).  Lane
// l takes the 16-byte output granules l, l + 32, ..., kCopyUnroll at a time with
// all their window loads issued before the first store, so that a warp keeps
// many loads in flight.
constexpr int kCopyUnroll = 2;

__device__ __forceinline__ void copy_coded(const uint8_t *win, uint32_t len, uint8_t *dst, int lane) {
  if (lane < int(kStateBytes / 16))
    reinterpret_cast<uint4 *>(dst)[lane] = __ldcg(reinterpret_cast<const uint4 *>(win) + lane);
  const uint32_t nbytes = len - kStateBytes;   // 2w
  const uint32_t S = uint32_t(kWin) - nbytes;  // first word's byte offset in the window
  const uint32_t mis = S & 15u;
  const uint32_t A0 = S - mis;
  const uint32_t ngran = (nbytes + 15) / 16;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  constexpr int U = kCopyUnroll;
  for (uint32_t j0 = 0; j0 < ngran; j0 += U * 32) {
    uint4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const uint32_t j = j0 + u * 32 + lane;
      const uint32_t a_off = A0 + 16 * j;
      a[u] = j < ngran ? __ldcg(reinterpret_cast<const uint4 *>(win + a_off)) : zero;
      b[u] = j < ngran && a_off + 16 < uint32_t(kWin)
                 ? __ldcg(reinterpret_cast<const uint4 *>(win + a_off + 16)) : zero;
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const uint32_t j = j0 + u * 32 + lane;
      if (j < ngran)
        st_cs_v4(dst + kStateBytes + 16 * j, keep16(extract16(a[u], b[u], mis), int(nbytes) - int(16 * j)));
    }
  }
}

// A raw chunk: its nsym coded bytes, extracted again from the input.
template <int DT>
__device__ void copy_raw(const uint8_t *in, uint64_t k, uint32_t nsym, uint8_t *dst, int lane) {
  const uint32_t ngran = uint32_t(round16(nsym) / 16);
  for (uint32_t gi = lane; gi < ngran; gi += 32) {
    const uint32_t v0 = gi * 16;
    const int keep = int(nsym - v0);
    uint4 e;
    if (is_fp8(DT)) {
      const uint8_t *src = in + k * kChunk;
      if (keep >= 16) {
        const uint4 a = ld_nc_v4(src + v0);
        e = make_uint4(fp8_code4(a.x), fp8_code4(a.y), fp8_code4(a.z), fp8_code4(a.w));
      } else {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        for (int q = 0; q < keep; q++) w[q / 4] |= fp8_code(src[v0 + q]) << (8 * (q % 4));
        e = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else if (DT != WC_FP32) {
      const uint16_t *src = reinterpret_cast<const uint16_t *>(in) + k * kChunk;
      uint32_t w[8];
      if (keep >= 16) {
        const uint4 a = ld_nc_v4(src + v0), b = ld_nc_v4(src + v0 + 8);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      } else {
#pragma unroll
        for (int q = 0; q < 8; q++) {
          const uint32_t lo = 2 * q < keep ? src[v0 + 2 * q] : 0u;
          const uint32_t hi = 2 * q + 1 < keep ? src[v0 + 2 * q + 1] : 0u;
          w[q] = lo | (hi << 16);
        }
      }
      e = keep16(make_uint4(code4<DT>(w[0], w[1]), code4<DT>(w[2], w[3]), code4<DT>(w[4], w[5]),
                            code4<DT>(w[6], w[7])), keep);
    } else {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(in) + k * kChunk;
      uint32_t u[16];
#pragma unroll
      for (int q = 0; q < 16; q++) u[q] = q < keep ? src[v0 + q] : 0u;
      uint32_t ee[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint32_t p01 = __byte_perm(u[4 * q] << 1, u[4 * q + 1] << 1, 0x0073);
        const uint32_t p23 = __byte_perm(u[4 * q + 2] << 1, u[4 * q + 3] << 1, 0x0073);
        ee[q] = __byte_perm(p01, p23, 0x5410);
      }
      e = keep16(make_uint4(ee[0], ee[1], ee[2], ee[3]), keep);
    }
    st_cs_v4(dst + v0, e);
  }
}

// Exclusive prefix (padded bytes of chunks 0 .. k-1) of chunk k of a tensor
// from the look-back words; false if a predecessor failed or the wait ran
// out.  Lane l reads the word of chunk j - l; the words before chunk 0 count
// as an inclusive prefix of 0.
__device__ bool lookback(const uint64_t *stat, uint64_t k, uint64_t &excl, int lane) {
  uint64_t sum = 0;
  int64_t j = int64_t(k) - 1;
  const uint64_t t0 = global_ns();
  while (j >= 0) {
    const int64_t idx = j - lane;
    const uint64_t v = idx >= 0 ? ld_acquire_u64(stat + idx) : kStatInc;
    const uint32_t fl = uint32_t(v >> 62);
    const uint32_t bad = __ballot_sync(0xffffffffu, fl == 3u);
    const uint32_t inc = __ballot_sync(0xffffffffu, fl == 2u);
    const uint32_t stop = __ballot_sync(0xffffffffu, fl == 0u) | bad;
    const int first_stop = stop ? __ffs(int(stop)) - 1 : 32;
    const int first_inc = inc ? __ffs(int(inc)) - 1 : 32;
    if (first_inc < first_stop) {
      sum += warp_sum_u64(lane <= first_inc ? (v & kStatVal) : 0);
      excl = sum;
      return true;
    }
    if (first_stop < 32 && ((bad >> first_stop) & 1u)) return false;
    sum += warp_sum_u64(lane < first_stop ? (v & kStatVal) : 0);
    j -= first_stop;
    if (first_stop == 0) {  // the nearest unread predecessor is still coding
      if (global_ns() - t0 > kWaitNs) return false;
      __nanosleep(512);     // leave the issue slots to the warps that code
    }
  }
  excl = sum;
  return true;
}

// What placing a warp's chunks needs of its tensor (passed by value to an
// out-of-line function, so that the coding loops keep their registers).
struct PlaceArgs {
  uint64_t *stat;         // look-back words
  const uint8_t *win0;    // window of chunk 0
  const uint8_t *in;      // the tensor's values
  uint8_t *out;           // the container
  uint64_t *out_size;
  uint64_t n, nc;
  uint64_t off_chunk_off, off_chunk_len, off_exp;
};

// After the warp has coded chunks kA (and kA + 1 if hasB): place them.
template <int DT>
__device__ __noinline__ void place_chunks(const PlaceArgs a, uint64_t kA, bool hasB, uint32_t lenA,
                                          uint32_t lenB) {
  const int lane = threadIdx.x & 31;
  const uint64_t padA = round16(lenA), padB = hasB ? round16(lenB) : 0;
  if (lane == 0) {
    st_release_u64(a.stat + kA, kStatAgg | padA);
    if (hasB) st_release_u64(a.stat + kA + 1, kStatAgg | padB);
  }
  uint64_t excl = 0;
  const bool ok = lookback(a.stat, kA, excl, lane);
  if (!ok) {
    if (lane == 0) {
      st_release_u64(a.stat + kA, kStatBad);
      if (hasB) st_release_u64(a.stat + kA + 1, kStatBad);
      *a.out_size = 0;
    }
    return;
  }
  if (lane == 0) {
    st_release_u64(a.stat + kA, kStatInc | (excl + padA));
    if (hasB) st_release_u64(a.stat + kA + 1, kStatInc | (excl + padA + padB));
  }
  uint64_t *choff = reinterpret_cast<uint64_t *>(a.out + a.off_chunk_off);
  uint32_t *chlen = reinterpret_cast<uint32_t *>(a.out + a.off_chunk_len);
  for (int c = 0; c < (hasB ? 2 : 1); c++) {
    const uint64_t k = kA + c;
    const uint32_t len = c ? lenB : lenA;
    const uint64_t off = excl + (c ? padA : 0);
    const uint32_t nsym = chunk_nsym(a.n, k);
    if (lane == 0) {
      choff[k] = off;
      chlen[k] = len;
    }
    uint8_t *dst = a.out + a.off_exp + off;
    if (len == nsym) copy_raw<DT>(a.in, k, nsym, dst, lane);
    else copy_coded(a.win0 + k * kWin, len, dst, lane);
    if (k + 1 == a.nc && lane == 0) {
      const uint64_t exp_bytes = off + round16(len);
      choff[a.nc] = exp_bytes;
      uint64_t *h64 = reinterpret_cast<uint64_t *>(a.out);
      h64[6] = exp_bytes;
      h64[7] = a.off_exp + exp_bytes;
      *a.out_size = a.off_exp + exp_bytes;
    }
  }
}

template <int DT, bool W>
__device__ __forceinline__ void code_and_place(const EncItem &it, const Layout &L, uint64_t kA, bool hasB,
                                               int warp, int lane) {
  CoderOut co{s_len[warp], kA, it.scratch + scratch_win_offset(L.nc)};
  code_warp<DT, W>(it, L, kA, hasB, warp, co);
  __syncwarp();
  const uint32_t lenA = s_len[warp][0], lenB = hasB ? s_len[warp][1] : 0u;
  PlaceArgs a;
  a.stat = reinterpret_cast<uint64_t *>(it.scratch + kScrStat);
  a.win0 = co.win0;
  a.in = it.in;
  a.out = it.out;
  a.out_size = it.out_size;
  a.n = it.n;
  a.nc = L.nc;
  a.off_chunk_off = L.off_chunk_off;
  a.off_chunk_len = L.off_chunk_len;
  a.off_exp = L.off_exp;
  place_chunks<DT>(a, kA, hasB, lenA, lenB);
}

__global__ void __launch_bounds__(kHistThreads, 2) k_hist(const __grid_constant__ EncParams p) {
  __shared__ __align__(16) uint32_t sh[256 * 32];  // [symbol][lane]
  __shared__ uint64_t red[kHistThreads / 32 + 1];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const uint32_t b = blockIdx.x;
  uint32_t lo = 0, hi = p.ntseg - 1;  // last segment starting at or before b
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (p.tseg_start[mid] <= b) lo = mid; else hi = mid - 1;
  }
  const EncItem &it = p.items[p.tseg_item[lo]];
  const uint64_t tile = b - p.tseg_start[lo];
  for (int i = tid; i < 256 * 32 / 4; i += kHistThreads)
    reinterpret_cast<uint4 *>(sh)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  count_tile<kHistThreads>(it, tile, sh);
  __syncthreads();
  uint64_t *ghist = reinterpret_cast<uint64_t *>(it.scratch + kScrHist);
  if (tid < 256) {
    uint32_t sum = 0;
#pragma unroll 8
    for (int j = 0; j < 32; j++) sum += sh[(tid << 5) | ((j + tid) & 31)];
    if (sum) atomicAdd(reinterpret_cast<unsigned long long *>(&ghist[tid]),
                       static_cast<unsigned long long>(sum));
    __threadfence();
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t *ctr = reinterpret_cast<uint32_t *>(it.scratch + kScrCtr);
    const uint64_t nc = num_chunks(it.n);
    const uint32_t nt = uint32_t((nc + kHistChunks - 1) / kHistChunks);
    s_last = (atomicAdd(&ctr[0], 1u) == nt - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  publish_table<kHistThreads>(it, red);
}

// Coding task: chunks [16 j, 16 j + 16) of item `it` (by value: the coding
// loops get the registers the task loop does not need).
__device__ __noinline__ void code_task(const EncItem it, uint64_t j) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);
  if (tid == 0) {
    const uint32_t *ready = reinterpret_cast<const uint32_t *>(it.scratch + kScrCtr) + 2;
    const uint64_t t0 = global_ns();
    uint32_t r = ld_acquire_u32(ready);
    while (r == 0 && global_ns() - t0 <= kWaitNs) {
      __nanosleep(256);
      r = ld_acquire_u32(ready);
    }
    s_flag = r;
  }
  __syncthreads();
  const uint32_t ready = s_flag;
  const uint64_t kA = j * kCoderChunks + 2 * warp;
  if (ready == 0) {  // no table (cannot happen after k_hist): the tensor fails
    if (kA < L.nc && lane == 0) {
      uint64_t *stat = reinterpret_cast<uint64_t *>(it.scratch + kScrStat);
      st_release_u64(stat + kA, kStatBad);
      if (kA + 1 < L.nc) st_release_u64(stat + kA + 1, kStatBad);
      *it.out_size = 0;
    }
    return;
  }
  s_tab[tid] = __ldcg(reinterpret_cast<const uint4 *>(it.scratch + kScrTab) + tid);
  s_bias[tid] = __ldcg(reinterpret_cast<const uint32_t *>(it.scratch + kScrBias) + tid);
  __syncthreads();
  if (kA >= L.nc) return;
  const bool hasB = kA + 1 < L.nc;
  const bool wide = ready == 2;
  if (dtype == WC_BF16) {
    if (wide) code_and_place<WC_BF16, true>(it, L, kA, hasB, warp, lane);
    else code_and_place<WC_BF16, false>(it, L, kA, hasB, warp, lane);
  } else if (dtype == WC_FP16) {
    if (wide) code_and_place<WC_FP16, true>(it, L, kA, hasB, warp, lane);
    else code_and_place<WC_FP16, false>(it, L, kA, hasB, warp, lane);
  } else if (dtype == WC_FP8E4M3) {
    if (wide) code_and_place<WC_FP8E4M3, true>(it, L, kA, hasB, warp, lane);
    else code_and_place<WC_FP8E4M3, false>(it, L, kA, hasB, warp, lane);
  } else if (dtype == WC_FP8E5M2) {
    if (wide) code_and_place<WC_FP8E5M2, true>(it, L, kA, hasB, warp, lane);
    else code_and_place<WC_FP8E5M2, false>(it, L, kA, hasB, warp, lane);
  } else if (wide) {
    code_and_place<WC_FP32, true>(it, L, kA, hasB, warp, lane);
  } else {
    code_and_place<WC_FP32, false>(it, L, kA, hasB, warp, lane);
  }
}

__global__ void __launch_bounds__(kCoderThreads, 4) k_encode(const __grid_constant__ EncParams p) {
  const int tid = threadIdx.x;
  uint32_t *ticket = reinterpret_cast<uint32_t *>(p.items[0].scratch + kScrCtr) + 3;
  for (;;) {
    if (tid == 0) s_task = atomicAdd(ticket, 1u);
    __syncthreads();
    const uint32_t t = s_task;
    if (t >= p.total_tasks) return;
    uint32_t lo = 0, hi = p.ncseg - 1;  // last segment starting at or before t
    while (lo < hi) {
      const uint32_t mid = (lo + hi + 1) >> 1;
      if (p.cseg_start[mid] <= t) lo = mid; else hi = mid - 1;
    }
    code_task(p.items[p.cseg_item[lo]], t - p.cseg_start[lo]);
    __syncthreads();  // the block is done with this task's shared memory
  }
}

int encode_blocks_per_sm() {
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_encode, kCoderThreads, 0) != cudaSuccess)
    return 0;
  return nb;
}

cudaError_t launch_prep(const EncParams &p, cudaStream_t s) {
  k_prep<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hist(const EncParams &p, cudaStream_t s) {
  if (p.total_tiles == 0) return cudaSuccess;
  k_hist<<<p.total_tiles, kHistThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_encode(const EncParams &p, int grid, cudaStream_t s) {
  if (p.total_tasks == 0) return cudaSuccess;
  const int g = int(p.total_tasks) < grid ? int(p.total_tasks) : grid;
  k_encode<<<g, kCoderThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
