// k_hist.cu -- encoder stage 1: container header, per-tensor exponent
// histogram, and the 12-bit frequency table.
//
//  k_prep   one block per tensor: clears the tensor's scratch counters and
//           writes the fixed header fields and the zero padding of the
//           container (everything that depends on n alone).
//  k_hist   one block per tile of up to 4 chunks: reads the values as
//           integers (a NaN payload is never touched as a float), counts the
//           coded bytes -- the 8-bit exponent of bf16 / fp32, the reordered
//           high byte of fp16, the exponent nibble of fp8 e4m3 ("PTWM" How it
//           works 1-2: after the bit reorder
//           the exponent leads a whole byte; "SMEF" pass3_streams.py) -- into a
//           shared-memory histogram with one column per lane (so the 32 lanes
//           of a warp never collide on an address), folds it into the tensor's
//           global histogram, and the last block of each tensor turns the
//           counts into the table.
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
#include "wc_block.cuh"
#include "wc_format.cuh"
#include "wc_planes.cuh"

namespace wc {

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_prep(const __grid_constant__ EncParams p) {
  const EncItem &it = p.items[blockIdx.x];
  const int tid = threadIdx.x;
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);
  uint8_t *out = it.out;

  uint64_t *hist = reinterpret_cast<uint64_t *>(it.scratch + kScrHist);
  uint32_t *ctr = reinterpret_cast<uint32_t *>(it.scratch + kScrCtr);
  hist[tid] = 0;
  if (tid < 4) ctr[tid] = 0;

  // table: all zero until the last histogram block writes it (n = 0 keeps it)
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
      const uint64_t raw_bytes = dtype == WC_FP8E4M3 ? (it.n + 1) / 2 : it.n;
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
constexpr int kHistThreads = 512;

// a word holds two 2-byte values (bf16 or fp16): count their coded bytes
template <int DT>
__device__ __forceinline__ void count_word16(uint32_t *sh, int lane, uint32_t w) {
  atomicAdd(&sh[(code_byte<DT>(w & 0xFFFFu) << 5) | lane], 1u);
  atomicAdd(&sh[(code_byte<DT>(w >> 16) << 5) | lane], 1u);
}
__device__ __forceinline__ void count_fp32_word(uint32_t *sh, int lane, uint32_t u) {
  atomicAdd(&sh[(((u >> 23) & 0xFFu) << 5) | lane], 1u);
}

// The last block of a tensor: counts -> table, published to the container
// header (u16 freq[256]) and to the coder's scratch entries.
__device__ void publish_table(const EncItem &it, uint64_t *red) {
  const int tid = threadIdx.x;
  const bool own = tid < 256;  // thread s owns symbol s
  const uint64_t n = it.n;
  const uint64_t *ghist = reinterpret_cast<const uint64_t *>(it.scratch + kScrHist);
  uint64_t c = own ? __ldcg(&ghist[tid]) : 0;
  uint64_t f = 0;
  if (c) {
    f = c * uint64_t(kProbScale) / n;
    if (f < 1) f = 1;
  }
  const int64_t d = int64_t(kProbScale) - int64_t(block_sum_u64<kHistThreads>(f, red));
  if (d > 0) {
    uint64_t key = c ? ((c << 8) | uint64_t(255 - tid)) : 0;
    uint64_t best = block_max_u64<kHistThreads>(key, red);
    if (own && tid == int(255 - (best & 0xFF))) f += uint64_t(d);
  } else if (d < 0) {
    const uint64_t k = uint64_t(-d);
    uint32_t lo = 1, hi = kProbScale;
    while (lo < hi) {  // smallest T in [1, 4096] with D(T) <= k
      uint32_t mid = (lo + hi) >> 1;
      uint64_t Dm = block_sum_u64<kHistThreads>(f > mid ? f - mid : 0, red);
      if (Dm <= k) hi = mid; else lo = mid + 1;
    }
    const uint32_t T = lo;
    const uint64_t DT = block_sum_u64<kHistThreads>(f > T ? f - T : 0, red);
    const uint64_t r = k - DT;
    const bool ge = own && f >= T;
    const uint64_t rank = block_excl_scan_u64<kHistThreads>(ge ? 1 : 0, red);
    if (ge) f = T - (rank < r ? 1 : 0);
  }
  const uint64_t cum = block_excl_scan_u64<kHistThreads>(f, red);
  // The coder divides the state x by f after renormalisation, when
  // x < f 2^20.  Narrow format (every f <= 2048): q = floor(x m / 2^k) with
  // k = 31 + c, c = ceil(log2 f), m = ceil(2^k / f) < 2^32, computed as
  // umulhi(x, m) >> (c - 1).  With e = m f - 2^k < f, the error term
  // x e / (f 2^k) < f 2^20 f / (f 2^(31 + c)) <= 1 / f when f <= 2^11, so the
  // floor is exact.  Wide format (some f > 2048): m = ceil(2^64 / f) as two
  // 32-bit halves, exact for every x < 2^32.  In both, f = 1 uses the all-ones
  // multiplier, which yields q = x - 1, repaid by bias += 4095.
  const bool wide = block_max_u64<kHistThreads>(f, red) > 2048;
  if (own) {
    const uint32_t ff = uint32_t(f);
    reinterpret_cast<uint16_t *>(it.out + kFreqOffset)[tid] = uint16_t(ff);
    uint4 e = make_uint4(0, 0, 0, 0);
    uint32_t bias = 0;
    if (ff) {
      bias = uint32_t(cum) + (ff == 1 ? kProbScale - 1 : 0);
      e.y = uint32_t((uint64_t(ff) << 20) - 1);  // renormalise while x > xmax
      e.z = kProbScale - ff;
      if (wide) {
        const uint64_t m = ff >= 2 ? (~uint64_t(0) / ff + 1) : ~uint64_t(0);
        e.x = uint32_t(m);
        e.w = uint32_t(m >> 32);
      } else {
        uint32_t m = 0xFFFFFFFFu, sh = 0;
        if (ff >= 2) {
          const uint32_t c = 32 - __clz(ff - 1);
          m = uint32_t(((uint64_t(1) << (31 + c)) - 1) / ff + 1);
          sh = c - 1;
        }
        e.x = m;
        e.w = sh | (bias << 5);
      }
    }
    reinterpret_cast<uint4 *>(it.scratch + kScrTab)[tid] = e;
    reinterpret_cast<uint32_t *>(it.scratch + kScrBias)[tid] = bias;
  }
  if (tid == 0) reinterpret_cast<uint32_t *>(it.scratch + kScrCtr)[2] = wide ? 1u : 0u;
}

// 16 values' worth of coded-byte counts (one group) from raw words.
template <int DT>
__device__ __forceinline__ void count_group16(uint32_t *sh, int lane, uint4 a, uint4 b) {
  count_word16<DT>(sh, lane, a.x); count_word16<DT>(sh, lane, a.y);
  count_word16<DT>(sh, lane, a.z); count_word16<DT>(sh, lane, a.w);
  count_word16<DT>(sh, lane, b.x); count_word16<DT>(sh, lane, b.y);
  count_word16<DT>(sh, lane, b.z); count_word16<DT>(sh, lane, b.w);
}

// fp8 e4m3: a word holds four values; count their exponent nibbles.
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

// One thread's share of a tile of fp8 values (16-value groups of 16 bytes).
__device__ __forceinline__ void count_tile8(uint32_t *sh, int lane, int tid, const uint8_t *src,
                                            uint32_t nfull, uint32_t count) {
  uint32_t g = tid;
  for (; g + 3 * kHistThreads < nfull; g += 4 * kHistThreads) {
    uint4 a0 = ld_nc_v4(src + 16 * g), a1 = ld_nc_v4(src + 16 * (g + kHistThreads));
    uint4 a2 = ld_nc_v4(src + 16 * (g + 2 * kHistThreads)), a3 = ld_nc_v4(src + 16 * (g + 3 * kHistThreads));
    count_quad8(sh, lane, a0);
    count_quad8(sh, lane, a1);
    count_quad8(sh, lane, a2);
    count_quad8(sh, lane, a3);
  }
  for (; g < nfull; g += kHistThreads) count_quad8(sh, lane, ld_nc_v4(src + 16 * g));
  if (g == nfull)  // the thread whose next group is the ragged tail
    for (uint32_t v = 16 * nfull; v < count; v++)
      atomicAdd(&sh[(fp8_code(src[v]) << 5) | lane], 1u);
}

// One thread's share of a tile of 2-byte values: groups tid, tid + 512, ...
// with four groups of loads in flight.
template <int DT>
__device__ __forceinline__ void count_tile16(uint32_t *sh, int lane, int tid, const uint16_t *src,
                                             uint32_t nfull, uint32_t count) {
  uint32_t g = tid;
  for (; g + 3 * kHistThreads < nfull; g += 4 * kHistThreads) {
    uint4 a0 = ld_nc_v4(src + 16 * g), b0 = ld_nc_v4(src + 16 * g + 8);
    uint4 a1 = ld_nc_v4(src + 16 * (g + kHistThreads)), b1 = ld_nc_v4(src + 16 * (g + kHistThreads) + 8);
    uint4 a2 = ld_nc_v4(src + 16 * (g + 2 * kHistThreads)), b2 = ld_nc_v4(src + 16 * (g + 2 * kHistThreads) + 8);
    uint4 a3 = ld_nc_v4(src + 16 * (g + 3 * kHistThreads)), b3 = ld_nc_v4(src + 16 * (g + 3 * kHistThreads) + 8);
    count_group16<DT>(sh, lane, a0, b0);
    count_group16<DT>(sh, lane, a1, b1);
    count_group16<DT>(sh, lane, a2, b2);
    count_group16<DT>(sh, lane, a3, b3);
  }
  for (; g < nfull; g += kHistThreads)
    count_group16<DT>(sh, lane, ld_nc_v4(src + 16 * g), ld_nc_v4(src + 16 * g + 8));
  if (g == nfull)  // the thread whose next group is the ragged tail
    for (uint32_t v = 16 * nfull; v < count; v++)
      atomicAdd(&sh[(code_byte<DT>(src[v]) << 5) | lane], 1u);
}
__device__ __forceinline__ void count_quad_fp32(uint32_t *sh, int lane, uint4 a) {
  count_fp32_word(sh, lane, a.x); count_fp32_word(sh, lane, a.y);
  count_fp32_word(sh, lane, a.z); count_fp32_word(sh, lane, a.w);
}

// One block counts a tile of up to kHistChunks chunks of one tensor.  Each
// thread takes 16-value groups tid, tid + 512, ... and keeps four groups of
// loads in flight.
__global__ void __launch_bounds__(kHistThreads, 2) k_hist(const __grid_constant__ EncParams p) {
  __shared__ __align__(16) uint32_t sh[256 * 32];  // [exponent][lane]
  __shared__ uint64_t red[kHistThreads / 32 + 1];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t b = blockIdx.x;
  const EncItem &it = p.items[find_item_by_hist(p, b)];
  const uint64_t tile = b - it.hist_base;
  const uint64_t v0 = tile * kHistChunks * kChunk;
  const uint64_t left = it.n - v0;
  const uint32_t count = uint32_t(left < uint64_t(kHistChunks) * kChunk ? left : uint64_t(kHistChunks) * kChunk);
  const uint64_t nc = num_chunks(it.n);
  const uint32_t nfull = count / 16;  // full 16-value groups

  for (int i = tid; i < 256 * 32 / 4; i += kHistThreads)
    reinterpret_cast<uint4 *>(sh)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();

  if (it.dtype == WC_BF16) {
    count_tile16<WC_BF16>(sh, lane, tid, reinterpret_cast<const uint16_t *>(it.in) + v0, nfull, count);
  } else if (it.dtype == WC_FP16) {
    count_tile16<WC_FP16>(sh, lane, tid, reinterpret_cast<const uint16_t *>(it.in) + v0, nfull, count);
  } else if (it.dtype == WC_FP8E4M3) {
    count_tile8(sh, lane, tid, it.in + v0, nfull, count);
  } else {
    const uint32_t *src = reinterpret_cast<const uint32_t *>(it.in) + v0;
    uint32_t g = tid;
    for (; g + kHistThreads < nfull; g += 2 * kHistThreads) {
      const uint32_t *s0 = src + 16 * g, *s1 = src + 16 * (g + kHistThreads);
      uint4 a0 = ld_nc_v4(s0), b0 = ld_nc_v4(s0 + 4), c0 = ld_nc_v4(s0 + 8), d0 = ld_nc_v4(s0 + 12);
      uint4 a1 = ld_nc_v4(s1), b1 = ld_nc_v4(s1 + 4), c1 = ld_nc_v4(s1 + 8), d1 = ld_nc_v4(s1 + 12);
      count_quad_fp32(sh, lane, a0); count_quad_fp32(sh, lane, b0);
      count_quad_fp32(sh, lane, c0); count_quad_fp32(sh, lane, d0);
      count_quad_fp32(sh, lane, a1); count_quad_fp32(sh, lane, b1);
      count_quad_fp32(sh, lane, c1); count_quad_fp32(sh, lane, d1);
    }
    for (; g < nfull; g += kHistThreads) {
      const uint32_t *s0 = src + 16 * g;
      count_quad_fp32(sh, lane, ld_nc_v4(s0)); count_quad_fp32(sh, lane, ld_nc_v4(s0 + 4));
      count_quad_fp32(sh, lane, ld_nc_v4(s0 + 8)); count_quad_fp32(sh, lane, ld_nc_v4(s0 + 12));
    }
    if (g == nfull)
      for (uint32_t v = 16 * nfull; v < count; v++) count_fp32_word(sh, lane, src[v]);
  }
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
    const uint32_t nb = uint32_t((nc + kHistChunks - 1) / kHistChunks);
    s_last = (atomicAdd(&ctr[0], 1u) == nb - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  publish_table(it, red);
}

cudaError_t launch_prep(const EncParams &p, cudaStream_t s) {
  k_prep<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hist(const EncParams &p, cudaStream_t s) {
  if (p.total_hist_blocks == 0) return cudaSuccess;
  k_hist<<<p.total_hist_blocks, kHistThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
