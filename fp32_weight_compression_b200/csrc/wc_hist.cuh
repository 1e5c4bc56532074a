// wc_hist.cuh -- the per-tensor histogram of coded bytes and the 12-bit
// frequency table built from it (device functions of the encoder).
//
// Counting: a block counts a tile of up to kHistChunks chunks of one tensor
// into a shared-memory histogram with one column per lane ([symbol][lane], so
// the 32 lanes of a warp never collide on an address), reading the values as
// integers (a NaN payload is never touched as a float).  The coded byte is the
// 8-bit exponent of bf16 / fp32, the reordered high byte of fp16, the high
// nibble of fp8 ("PTWM" How it works 1-2: after the bit reorder the exponent
// leads; "SMEF" pass3_streams.py).  The tile's counts are added into the
// tensor's global histogram; the last tile of a tensor turns the counts into
// the table.
//
// Table rule (the pages fix none; this is the container's rule):
// f_s = 0 if c_s = 0 else max(1, floor(c_s 4096 / n));
// d = 4096 - sum f; d > 0: the symbol with the largest count (lowest symbol on
// ties) takes d; d < 0: -d times the symbol with the largest f among f > 1
// (lowest symbol on ties) gives up one.  The repeated give-up is evaluated in
// closed form here: with D(T) = sum max(0, f_s - T), let T be the smallest
// level >= 1 with D(T) <= -d; every f_s >= T becomes T, and the r = -d - D(T)
// lowest-numbered of them go on to T - 1.  This is the state the one-at-a-time
// rule reaches: it always lowers a current maximum, so it flattens everything
// above T to T first, and then takes the tied symbols at T in symbol order.
#pragma once

#include "wc_block.cuh"
#include "wc_coder.cuh"
#include "wc_format.cuh"
#include "wc_planes.cuh"

namespace wc {

// a word holds two 2-byte values (bf16 or fp16): count their coded bytes
template <int DT>
__device__ __forceinline__ void count_word16(uint32_t *sh, int lane, uint32_t w) {
  atomicAdd(&sh[(code_byte<DT>(w & 0xFFFFu) << 5) | lane], 1u);
  atomicAdd(&sh[(code_byte<DT>(w >> 16) << 5) | lane], 1u);
}
__device__ __forceinline__ void count_fp32_word(uint32_t *sh, int lane, uint32_t u) {
  atomicAdd(&sh[(((u >> 23) & 0xFFu) << 5) | lane], 1u);
}

// 16 values' worth of coded-byte counts (one group) from raw words.
template <int DT>
__device__ __forceinline__ void count_group16(uint32_t *sh, int lane, uint4 a, uint4 b) {
  count_word16<DT>(sh, lane, a.x); count_word16<DT>(sh, lane, a.y);
  count_word16<DT>(sh, lane, a.z); count_word16<DT>(sh, lane, a.w);
  count_word16<DT>(sh, lane, b.x); count_word16<DT>(sh, lane, b.y);
  count_word16<DT>(sh, lane, b.z); count_word16<DT>(sh, lane, b.w);
}

// fp8: a word holds four values; count their coded nibbles.
__device__ __forceinline__ void count_word8(uint32_t *sh, int lane, uint32_t w) {
  atomicAdd(&sh[(fp8_code(w) << 5) | lane], 1u);
  atomicAdd(&sh[(fp8_code(w >> 8) << 5) | lane], 1u);
  atomicAdd(&sh[(fp8_code(w >> 16) << 5) | lane], 1u);
  atomicAdd(&sh[(fp8_code(w >> 24) << 5) | lane], 1u);
}
__device__ __forceinline__ void count_quad8(uint32_t *sh, int lane, uint4 a) {
  count_word8(sh, lane, a.x); count_word8(sh, lane, a.y);
  count_word8(sh, lane, a.z); count_word8(sh, lane, a.w);
}
__device__ __forceinline__ void count_quad_fp32(uint32_t *sh, int lane, uint4 a) {
  count_fp32_word(sh, lane, a.x); count_fp32_word(sh, lane, a.y);
  count_fp32_word(sh, lane, a.z); count_fp32_word(sh, lane, a.w);
}

// One thread's share of a tile of fp8 values (16-value groups of 16 bytes):
// groups tid, tid + NT, ... with four groups of loads in flight.
template <int NT>
__device__ __forceinline__ void count_tile8(uint32_t *sh, int lane, int tid, const uint8_t *src,
                                            uint32_t nfull, uint32_t count) {
  uint32_t g = tid;
  for (; g + 3 * NT < nfull; g += 4 * NT) {
    uint4 a0 = ld_nc_v4(src + 16 * g), a1 = ld_nc_v4(src + 16 * (g + NT));
    uint4 a2 = ld_nc_v4(src + 16 * (g + 2 * NT)), a3 = ld_nc_v4(src + 16 * (g + 3 * NT));
    count_quad8(sh, lane, a0);
    count_quad8(sh, lane, a1);
    count_quad8(sh, lane, a2);
    count_quad8(sh, lane, a3);
  }
  for (; g < nfull; g += NT) count_quad8(sh, lane, ld_nc_v4(src + 16 * g));
  if (g == nfull)  // the thread whose next group is the ragged tail
    for (uint32_t v = 16 * nfull; v < count; v++)
      atomicAdd(&sh[(fp8_code(src[v]) << 5) | lane], 1u);
}

// 2-byte values (bf16 / fp16), as count_tile8.
template <int DT, int NT>
__device__ __forceinline__ void count_tile16(uint32_t *sh, int lane, int tid, const uint16_t *src,
                                             uint32_t nfull, uint32_t count) {
  uint32_t g = tid;
  for (; g + 3 * NT < nfull; g += 4 * NT) {
    uint4 a0 = ld_nc_v4(src + 16 * g), b0 = ld_nc_v4(src + 16 * g + 8);
    uint4 a1 = ld_nc_v4(src + 16 * (g + NT)), b1 = ld_nc_v4(src + 16 * (g + NT) + 8);
    uint4 a2 = ld_nc_v4(src + 16 * (g + 2 * NT)), b2 = ld_nc_v4(src + 16 * (g + 2 * NT) + 8);
    uint4 a3 = ld_nc_v4(src + 16 * (g + 3 * NT)), b3 = ld_nc_v4(src + 16 * (g + 3 * NT) + 8);
    count_group16<DT>(sh, lane, a0, b0);
    count_group16<DT>(sh, lane, a1, b1);
    count_group16<DT>(sh, lane, a2, b2);
    count_group16<DT>(sh, lane, a3, b3);
  }
  for (; g < nfull; g += NT)
    count_group16<DT>(sh, lane, ld_nc_v4(src + 16 * g), ld_nc_v4(src + 16 * g + 8));
  if (g == nfull)
    for (uint32_t v = 16 * nfull; v < count; v++)
      atomicAdd(&sh[(code_byte<DT>(src[v]) << 5) | lane], 1u);
}

// fp32 values, two groups of loads in flight.
template <int NT>
__device__ __forceinline__ void count_tile32(uint32_t *sh, int lane, int tid, const uint32_t *src,
                                             uint32_t nfull, uint32_t count) {
  uint32_t g = tid;
  for (; g + NT < nfull; g += 2 * NT) {
    const uint32_t *s0 = src + 16 * g, *s1 = src + 16 * (g + NT);
    uint4 a0 = ld_nc_v4(s0), b0 = ld_nc_v4(s0 + 4), c0 = ld_nc_v4(s0 + 8), d0 = ld_nc_v4(s0 + 12);
    uint4 a1 = ld_nc_v4(s1), b1 = ld_nc_v4(s1 + 4), c1 = ld_nc_v4(s1 + 8), d1 = ld_nc_v4(s1 + 12);
    count_quad_fp32(sh, lane, a0); count_quad_fp32(sh, lane, b0);
    count_quad_fp32(sh, lane, c0); count_quad_fp32(sh, lane, d0);
    count_quad_fp32(sh, lane, a1); count_quad_fp32(sh, lane, b1);
    count_quad_fp32(sh, lane, c1); count_quad_fp32(sh, lane, d1);
  }
  for (; g < nfull; g += NT) {
    const uint32_t *s0 = src + 16 * g;
    count_quad_fp32(sh, lane, ld_nc_v4(s0)); count_quad_fp32(sh, lane, ld_nc_v4(s0 + 4));
    count_quad_fp32(sh, lane, ld_nc_v4(s0 + 8)); count_quad_fp32(sh, lane, ld_nc_v4(s0 + 12));
  }
  if (g == nfull)
    for (uint32_t v = 16 * nfull; v < count; v++) count_fp32_word(sh, lane, src[v]);
}

// Count tile `tile` of item `it` (all NT threads of the block) into sh
// (256 x 32 u32, zeroed by the caller).
template <int NT>
__device__ __forceinline__ void count_tile(const EncItem &it, uint64_t tile, uint32_t *sh) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint64_t v0 = tile * kHistChunks * kChunk;
  const uint64_t left = it.n - v0;
  const uint32_t count =
      uint32_t(left < uint64_t(kHistChunks) * kChunk ? left : uint64_t(kHistChunks) * kChunk);
  const uint32_t nfull = count / 16;  // full 16-value groups
  const int dt = int(it.dtype);
  if (dt == WC_BF16) {
    count_tile16<WC_BF16, NT>(sh, lane, tid, reinterpret_cast<const uint16_t *>(it.in) + v0, nfull, count);
  } else if (dt == WC_FP16) {
    count_tile16<WC_FP16, NT>(sh, lane, tid, reinterpret_cast<const uint16_t *>(it.in) + v0, nfull, count);
  } else if (is_fp8(dt)) {
    count_tile8<NT>(sh, lane, tid, it.in + v0, nfull, count);
  } else {
    count_tile32<NT>(sh, lane, tid, reinterpret_cast<const uint32_t *>(it.in) + v0, nfull, count);
  }
}

// The last block of a tensor: counts -> table, published to the container
// header (u16 freq[256]) and to the coder's scratch entries.  Every thread of
// the block calls it; thread s < 256 owns symbol s.
template <int NT>
__device__ void publish_table(const EncItem &it, uint64_t *red) {
  const int tid = threadIdx.x;
  const bool own = tid < 256;
  const uint64_t n = it.n;
  const uint64_t *ghist = reinterpret_cast<const uint64_t *>(it.scratch + kScrHist);
  uint64_t c = own ? __ldcg(&ghist[tid]) : 0;
  uint64_t f = 0;
  if (c) {
    f = c * uint64_t(kProbScale) / n;
    if (f < 1) f = 1;
  }
  const int64_t d = int64_t(kProbScale) - int64_t(block_sum_u64<NT>(f, red));
  if (d > 0) {
    uint64_t key = c ? ((c << 8) | uint64_t(255 - tid)) : 0;
    uint64_t best = block_max_u64<NT>(key, red);
    if (own && tid == int(255 - (best & 0xFF))) f += uint64_t(d);
  } else if (d < 0) {
    const uint64_t k = uint64_t(-d);
    uint32_t lo = 1, hi = kProbScale;
    while (lo < hi) {  // smallest T in [1, 4096] with D(T) <= k
      uint32_t mid = (lo + hi) >> 1;
      uint64_t Dm = block_sum_u64<NT>(f > mid ? f - mid : 0, red);
      if (Dm <= k) hi = mid; else lo = mid + 1;
    }
    const uint32_t T = lo;
    const uint64_t DT = block_sum_u64<NT>(f > T ? f - T : 0, red);
    const uint64_t r = k - DT;
    const bool ge = own && f >= T;
    const uint64_t rank = block_excl_scan_u64<NT>(ge ? 1 : 0, red);
    if (ge) f = T - (rank < r ? 1 : 0);
  }
  const uint64_t cum = block_excl_scan_u64<NT>(f, red);
  const bool wide = block_max_u64<NT>(f, red) > 2048;
  if (own) {
    const uint32_t ff = uint32_t(f);
    reinterpret_cast<uint16_t *>(it.out + kFreqOffset)[tid] = uint16_t(ff);
    uint4 e;
    uint32_t bias;
    coder_entry(ff, uint32_t(cum), wide, e, bias);
    reinterpret_cast<uint4 *>(it.scratch + kScrTab)[tid] = e;
    reinterpret_cast<uint32_t *>(it.scratch + kScrBias)[tid] = bias;
  }
  // the table is complete once every owner's stores are visible; then the
  // ready word (1 narrow, 2 wide) is released to the coding blocks
  __threadfence();
  __syncthreads();
  if (tid == 0) st_release_u32(reinterpret_cast<uint32_t *>(it.scratch + kScrCtr) + 2, wide ? 2u : 1u);
}

}  // namespace wc
