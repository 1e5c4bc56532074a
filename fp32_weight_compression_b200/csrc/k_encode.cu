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
// two 32-bit halves (wc_coder.cuh); the coder is compiled for both and each
// block takes the form its tensor's table was written in.  The lanes
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
#include "wc_planes.cuh"

namespace wc {

constexpr int kCoderThreads = kCoderWarps * 32;

// Per-block shared state of the coder, at namespace scope so that helper
// functions reach it as shared memory (not through generic pointers).
__shared__ uint4 s_tab[256];
__shared__ uint32_t s_bias[256];
__shared__ __align__(16) uint8_t s_ebuf[kCoderWarps][2][kGroupValues];

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
  uint32_t *lens;
  uint8_t *win0;  // window of chunk 0 of the tensor
};

__device__ __forceinline__ void finish_chunk(const CoderOut &co, uint64_t k, uint32_t nsym, uint32_t x,
                                             uint32_t tail, bool bail, int lane) {
  const uint32_t w = kWinWords - tail;
  const bool raw = bail || (kStateBytes + 2 * w >= nsym);
  const uint32_t len = raw ? nsym : kStateBytes + 2 * w;
  if (!raw) reinterpret_cast<uint32_t *>(co.win0 + k * kWin)[lane] = x;
  if (lane == 0) co.lens[k] = len;
}

// Two full 2-byte-value chunks (bf16 or fp16) kA, kA + 1 in lock-step.
template <int DT, bool W>
__device__ void code_pair16(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
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
__device__ void code_pair_fp32(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
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
__device__ void code_pair8(const EncItem &it, const Layout &L, uint64_t kA, const uint4 *tab,
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

__global__ void __launch_bounds__(kCoderThreads, 4) k_coder(const __grid_constant__ EncParams p) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t b = blockIdx.x;
  const EncItem &it = p.items[find_item_by_block(p, b)];
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);

  s_tab[tid] = reinterpret_cast<const uint4 *>(it.scratch + kScrTab)[tid];
  s_bias[tid] = reinterpret_cast<const uint32_t *>(it.scratch + kScrBias)[tid];
  __syncthreads();

  const uint64_t kA = uint64_t(b - it.block_base) * kCoderChunks + 2 * warp;
  if (kA >= L.nc) return;
  const bool hasB = kA + 1 < L.nc;
  CoderOut co{reinterpret_cast<uint32_t *>(it.scratch + kScrLen), it.scratch + scratch_win_offset(L.nc)};
  const bool wide = reinterpret_cast<const uint32_t *>(it.scratch + kScrCtr)[2] == 2;
  if (dtype == WC_BF16) {
    if (wide) code_warp<WC_BF16, true>(it, L, kA, hasB, warp, co);
    else code_warp<WC_BF16, false>(it, L, kA, hasB, warp, co);
  } else if (dtype == WC_FP16) {
    if (wide) code_warp<WC_FP16, true>(it, L, kA, hasB, warp, co);
    else code_warp<WC_FP16, false>(it, L, kA, hasB, warp, co);
  } else if (dtype == WC_FP8E4M3) {
    if (wide) code_warp<WC_FP8E4M3, true>(it, L, kA, hasB, warp, co);
    else code_warp<WC_FP8E4M3, false>(it, L, kA, hasB, warp, co);
  } else if (dtype == WC_FP8E5M2) {
    if (wide) code_warp<WC_FP8E5M2, true>(it, L, kA, hasB, warp, co);
    else code_warp<WC_FP8E5M2, false>(it, L, kA, hasB, warp, co);
  } else if (wide) {
    code_warp<WC_FP32, true>(it, L, kA, hasB, warp, co);
  } else {
    code_warp<WC_FP32, false>(it, L, kA, hasB, warp, co);
  }

  // last warp of the tensor: offset table and the rest of the header
  const uint32_t done = hasB ? 2u : 1u;
  __threadfence();
  uint32_t prev = 0;
  if (lane == 0) prev = atomicAdd(reinterpret_cast<uint32_t *>(it.scratch + kScrCtr) + 1, done);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev + done != uint32_t(L.nc)) return;
  __threadfence();
  const uint32_t *lens = co.lens;
  uint64_t *choff = reinterpret_cast<uint64_t *>(it.out + L.off_chunk_off);
  uint32_t *chlen = reinterpret_cast<uint32_t *>(it.out + L.off_chunk_len);
  uint64_t run = 0;
  for (uint64_t base = 0; base < L.nc; base += 32) {
    const uint64_t j = base + lane;
    const uint32_t ln = j < L.nc ? __ldcg(&lens[j]) : 0u;
    const uint64_t pd = round16(ln);
    const uint64_t incl = warp_incl_scan_u64(pd);
    if (j < L.nc) {
      choff[j] = run + incl - pd;
      chlen[j] = ln;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    choff[L.nc] = run;
    uint64_t *h64 = reinterpret_cast<uint64_t *>(it.out);
    h64[6] = run;
    h64[7] = L.off_exp + run;
    *it.out_size = L.off_exp + run;
  }
}

cudaError_t launch_coder(const EncParams &p, cudaStream_t s) {
  if (p.total_coder_blocks == 0) return cudaSuccess;
  k_coder<<<p.total_coder_blocks, kCoderThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
