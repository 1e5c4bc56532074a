// k_split12.cu -- the Split12 serving format for bf16 (include/wc_split12.h;
// "weight-compression" README: the high byte from a codebook, the low byte
// raw): encoder in six kernels, decoder in one, and their C ABI.
//
// Encode (all on one stream, sizes from n alone):
//   k12_prep   1 block    header fields that depend on n, zero padding,
//                         clears the global high-byte histogram
//   k12_hist   1 block / chunk   high-byte counts of the chunk (one column
//                         per lane in shared memory), kept per chunk and
//                         added to the global histogram
//   k12_book   1 block    the 16 most frequent high bytes (ties to the smaller
//                         byte), ascending -> codebook, K, and a 256-entry
//                         byte -> slot table (0xFF: missed)
//   k12_count  1 warp / chunk   the chunk's exceptions from its histogram
//   k12_scan   1 block    exclusive scan -> exc_off[], ne, total size, the
//                         padding after the exception lists
//   k12_pack   1 block / chunk   index nibbles and low bytes, a warp per
//                         eighth of the chunk; exceptions in ascending
//                         position at the chunk's exc_off
// Decode: k12_decode, one block per chunk:
// expands 16 values per thread per step (the codebook lives in four
// registers; byte permutes do the lookup), then patches the chunk's
// exceptions after a block barrier.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "wc.h"
#include "wc_block.cuh"
#include "wc_split12.cuh"

namespace wc12 {

__device__ __forceinline__ void report(int32_t *status, int32_t code) { atomicCAS(status, 0, code); }

// Launch parameters of a batch (up to kBatchMax tensors per launch; passed by
// value).  Encode: the kernels that work per chunk find their tensor by its
// first chunk (chunk_base), k12_count by its first block (count_base); the
// per-tensor kernels take one block per tensor.
constexpr uint32_t kBatchMax = 256;
struct EncItem12 {
  const uint16_t *in;
  uint8_t *out;
  uint8_t *scr;
  uint64_t *out_size;
  uint64_t n;
  uint32_t chunk_base;
  uint32_t count_base;
};
struct EncBatch12 {
  uint32_t count, total_chunks, total_count_blocks, pad;
  EncItem12 items[kBatchMax];
};
struct DecItem12 {
  const uint8_t *cont;
  uint64_t cont_bytes;
  uint16_t *out;
  uint64_t n;         // the values the caller expects (the header must agree)
  uint32_t unit_base; // first work unit: one per chunk, one for an empty tensor
  uint32_t pad;
};
struct DecBatch12 {
  uint32_t count, total_units;
  int32_t *status;
  DecItem12 items[kBatchMax];
};

template <typename Item, typename F>
__device__ __forceinline__ uint32_t find_item(const Item *items, uint32_t count, uint32_t g, F base_of) {
  uint32_t lo = 0, hi = count - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (base_of(items[mid]) <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k12_prep(const __grid_constant__ EncBatch12 b) {
  const EncItem12 &it = b.items[blockIdx.x];
  const uint64_t n = it.n;
  uint8_t *out = it.out, *scr = it.scr;
  const int tid = threadIdx.x;
  const Lay L = lay(n, 0);
  reinterpret_cast<unsigned long long *>(scr + kScrHist)[tid] = 0;
  if (tid == 0) {
    uint32_t *h32 = reinterpret_cast<uint32_t *>(out);
    uint64_t *h64 = reinterpret_cast<uint64_t *>(out);
    h32[0] = kMagic;
    h32[1] = 1u | (1u << 16);  // version 1, dtype bf16; K follows from k12_book
    h64[1] = n;
    h32[4] = uint32_t(kChunk);
    h32[5] = uint32_t(L.nc);
    h64[3] = 0;                // ne: k12_scan
    h64[4] = L.off_idx;
    h64[5] = L.off_lo;
    h64[6] = L.off_exc;
    h64[7] = 0;                // total: k12_scan
  }
  // padding that depends on n alone (each run is shorter than 16 bytes)
  const uint64_t z0 = kExcOffOff + 8 * (L.nc + 1), z1 = L.off_idx + (n + 1) / 2, z2 = L.off_lo + n;
  if (tid < 16) {
    if (z0 + tid < L.off_idx) out[z0 + tid] = 0;
  } else if (tid < 32) {
    if (z1 + (tid - 16) < L.off_lo) out[z1 + (tid - 16)] = 0;
  } else if (tid < 48) {
    if (z2 + (tid - 32) < L.off_exc) out[z2 + (tid - 32)] = 0;
  }
}

// ---------------------------------------------------------------------------
constexpr int kHistThreads = 512;

__device__ __forceinline__ void count_hi(uint32_t *sh, int lane, uint32_t w) {
  atomicAdd(&sh[(((w >> 8) & 0xFFu) << 5) | lane], 1u);
  atomicAdd(&sh[((w >> 24) << 5) | lane], 1u);
}

__device__ __forceinline__ void count_group(uint32_t *sh, int lane, uint4 a, uint4 b) {
  count_hi(sh, lane, a.x); count_hi(sh, lane, a.y); count_hi(sh, lane, a.z); count_hi(sh, lane, a.w);
  count_hi(sh, lane, b.x); count_hi(sh, lane, b.y); count_hi(sh, lane, b.z); count_hi(sh, lane, b.w);
}

__global__ void __launch_bounds__(kHistThreads, 2) k12_hist(const __grid_constant__ EncBatch12 b) {
  __shared__ __align__(16) uint32_t sh[256 * 32];  // [high byte][lane]
  const EncItem12 &it =
      b.items[find_item(b.items, b.count, blockIdx.x, [](const EncItem12 &x) { return x.chunk_base; })];
  const uint16_t *__restrict__ in = it.in;
  const uint64_t n = it.n;
  uint8_t *scr = it.scr;
  const int tid = threadIdx.x, lane = tid & 31;
  const uint64_t c = blockIdx.x - it.chunk_base, v0 = c * kChunk;
  const uint32_t count = uint32_t(n - v0 < kChunk ? n - v0 : kChunk);
  const uint32_t nfull = count / 16;
  for (int i = tid; i < 256 * 32 / 4; i += kHistThreads)
    reinterpret_cast<uint4 *>(sh)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  const uint16_t *src = in + v0;
  uint32_t g = tid;
  for (; g + kHistThreads < nfull; g += 2 * kHistThreads) {
    const uint16_t *s0 = src + 16 * g, *s1 = src + 16 * (g + kHistThreads);
    const uint4 a0 = wc::ld_nc_v4(s0), b0 = wc::ld_nc_v4(s0 + 8);
    const uint4 a1 = wc::ld_nc_v4(s1), b1 = wc::ld_nc_v4(s1 + 8);
    count_group(sh, lane, a0, b0);
    count_group(sh, lane, a1, b1);
  }
  for (; g < nfull; g += kHistThreads)
    count_group(sh, lane, wc::ld_nc_v4(src + 16 * g), wc::ld_nc_v4(src + 16 * g + 8));
  if (g == nfull)  // the thread whose next group is the ragged tail
    for (uint32_t v = 16 * nfull; v < count; v++) atomicAdd(&sh[((uint32_t(src[v]) >> 8) << 5) | lane], 1u);
  __syncthreads();
  if (tid < 256) {
    uint32_t sum = 0;
#pragma unroll 8
    for (int j = 0; j < 32; j++) sum += sh[(tid << 5) | ((j + tid) & 31)];
    reinterpret_cast<uint32_t *>(scr + kScrChunkHist)[c * 256 + tid] = sum;
    if (sum)
      atomicAdd(reinterpret_cast<unsigned long long *>(scr + kScrHist) + tid,
                static_cast<unsigned long long>(sum));
  }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k12_book(const __grid_constant__ EncBatch12 b) {
  uint8_t *out = b.items[blockIdx.x].out, *scr = b.items[blockIdx.x].scr;
  __shared__ unsigned long long cnt[256];
  __shared__ uint32_t wsel[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cnt[tid] = reinterpret_cast<const unsigned long long *>(scr + kScrHist)[tid];
  __syncthreads();
  const unsigned long long mine = cnt[tid];
  uint32_t rank = 0;  // bytes that beat this one: more values, or as many and smaller
  for (int b = 0; b < 256; b++) {
    const unsigned long long o = cnt[b];
    rank += (o > mine || (o == mine && b < tid)) ? 1u : 0u;
  }
  const bool sel = mine > 0 && rank < 16;
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, sel);
  if (lane == 0) wsel[warp] = __popc(bal);
  __syncthreads();
  uint32_t before = 0, k = 0;
  for (int w = 0; w < 8; w++) {
    before += w < warp ? wsel[w] : 0;
    k += wsel[w];
  }
  const uint32_t pos = before + __popc(bal & ((1u << lane) - 1u));
  scr[kScrLut + tid] = sel ? uint8_t(pos) : uint8_t(0xFF);
  if (sel) out[kBookOff + pos] = uint8_t(tid);
  if (tid < 16 && uint32_t(tid) >= k) out[kBookOff + tid] = 0;
  if (tid == 0) out[7] = uint8_t(k);
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k12_count(const __grid_constant__ EncBatch12 b) {
  __shared__ uint8_t lut[256];
  const EncItem12 &it =
      b.items[find_item(b.items, b.count, blockIdx.x, [](const EncItem12 &x) { return x.count_base; })];
  const uint64_t nc = (it.n + kChunk - 1) / kChunk;
  uint8_t *out = it.out;
  const uint8_t *scr = it.scr;
  const uint32_t lb = blockIdx.x - it.count_base;  // block of this tensor
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  lut[tid] = scr[kScrLut + tid];
  __syncthreads();
  const uint64_t c = uint64_t(lb) * 8 + warp;
  uint64_t *exc_off = reinterpret_cast<uint64_t *>(out + kExcOffOff);
  if (lb == 0 && tid == 0) exc_off[0] = 0;
  if (c >= nc) return;
  const uint32_t *h = reinterpret_cast<const uint32_t *>(scr + kScrChunkHist) + c * 256;
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 8; j++) {
    const int b = lane * 8 + j;
    s += lut[b] == 0xFF ? h[b] : 0u;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) exc_off[c + 1] = s;  // this chunk's count; k12_scan sums
}

// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) k12_scan(const __grid_constant__ EncBatch12 b) {
  const uint64_t n = b.items[blockIdx.x].n;
  uint8_t *out = b.items[blockIdx.x].out;
  uint64_t *out_size = b.items[blockIdx.x].out_size;
  __shared__ uint64_t red[kScanThreads / 32 + 1];
  __shared__ uint64_t s_ne;
  const int tid = threadIdx.x;
  const uint64_t nc = (n + kChunk - 1) / kChunk;
  uint64_t *exc_off = reinterpret_cast<uint64_t *>(out + kExcOffOff);
  uint64_t carry = 0;
  for (uint64_t base = 1; base <= nc; base += kScanThreads) {  // entries 1..nc, in place
    const uint64_t i = base + tid;
    const uint64_t v = i <= nc ? exc_off[i] : 0;
    const uint64_t ex = wc::block_excl_scan_u64<kScanThreads>(v, red);
    const uint64_t tot = wc::block_sum_u64<kScanThreads>(v, red);
    if (i <= nc) exc_off[i] = carry + ex + v;
    carry += tot;
  }
  if (tid == 0) s_ne = carry;
  __syncthreads();
  const uint64_t ne = s_ne;
  const Lay L = lay(n, ne);
  if (tid == 0) {
    uint64_t *h64 = reinterpret_cast<uint64_t *>(out);
    h64[3] = ne;
    h64[7] = L.total;
    *out_size = L.total;
  }
  const uint64_t z0 = L.off_exc + 2 * ne, z1 = L.off_excval + ne;
  if (tid < 16) {
    if (z0 + tid < L.off_excval) out[z0 + tid] = 0;
  } else if (tid < 32) {
    if (z1 + (tid - 16) < L.total) out[z1 + (tid - 16)] = 0;
  }
}

// ---------------------------------------------------------------------------
constexpr int kPackThreads = 256;

// slot of each of the 4 values' high bytes in byte j of the result
__device__ __forceinline__ uint32_t slots4(const uint8_t *lut, uint32_t w0, uint32_t w1) {
  const uint32_t hb = __byte_perm(w0, w1, 0x7531);
  return uint32_t(lut[hb & 0xFFu]) | (uint32_t(lut[(hb >> 8) & 0xFFu]) << 8) |
         (uint32_t(lut[(hb >> 16) & 0xFFu]) << 16) | (uint32_t(lut[hb >> 24]) << 24);
}

// 4 slots (bytes, 0xFF = missed) -> 4 index nibbles in the low 16 bits, and
// the number missed
__device__ __forceinline__ uint32_t nibbles4(uint32_t s4, uint32_t &missed) {
  const uint32_t miss = s4 & 0x80808080u;  // slots are < 16 or 0xFF
  missed += __popc(miss);
  const uint32_t idx = s4 & ~((miss >> 7) * 0xFFu);  // missed -> 0
  return (idx & 0xFu) | ((idx >> 4) & 0xF0u) | ((idx >> 8) & 0xF00u) | ((idx >> 12) & 0xF000u);
}

// The values of group g (16 values, or the chunk's ragged tail) that the
// codebook misses, in ascending position: fn(position in the chunk, high
// byte), for the first `missed` of them.
template <typename F>
__device__ __forceinline__ void for_misses(const uint8_t *lut, const uint16_t *src, uint32_t g, uint32_t nfull,
                                           uint32_t tail, const uint4 &a, const uint4 &b, uint32_t missed,
                                           F fn) {
  const uint32_t nv = g < nfull ? 16u : (g == nfull ? tail : 0u);
  for (uint32_t j = 0; j < nv && missed; j++) {
    uint32_t v;
    if (g < nfull) {
      const uint32_t w = j < 8 ? (&a.x)[j >> 1] : (&b.x)[(j - 8) >> 1];
      v = (j & 1) ? (w >> 16) : (w & 0xFFFFu);
    } else {
      v = src[16 * g + j];
    }
    const uint32_t h = v >> 8;
    if (lut[h] == 0xFFu) {
      fn(16 * g + j, h);
      missed--;
    }
  }
}

// exclusive prefix over the warp's lanes, and the warp's total
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t &total) {
  const int lane = threadIdx.x & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - v;
}

// Warp w of a block takes the chunk's groups [512 w, 512 (w + 1)), 32 a step
// (16 values a lane), so the warps run without block barriers: a warp's
// exceptions come in ascending position and are staged in shared memory;
// after the chunk, one barrier gives each warp the count of the warps before
// it, and the staged entries go to the chunk's list at that offset.  A warp
// with more than kStaged reads its range again and writes them in place.
constexpr uint32_t kPackWarps = kPackThreads / 32;
constexpr uint32_t kWarpGroups = kChunk / 16 / kPackWarps;  // 512
constexpr uint32_t kStaged = 256;

// A warp's exceptions written in place, in ascending position from
// exc_pos[e0] on, by reading its groups [g0, g1) again (the path for more
// than fit in the staging list).
__device__ __noinline__ void rewrite_misses(const uint8_t *lut, const uint16_t *src, uint32_t g0, uint32_t g1,
                                            uint32_t nfull, uint32_t tail, uint64_t e0, uint16_t *exc_pos,
                                            uint8_t *exc_val) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t r = 0;
  for (uint32_t gs = g0; gs < g1; gs += 32) {
    const uint32_t g = gs + lane;
    uint32_t missed = 0;
    uint4 a = make_uint4(0, 0, 0, 0), bq = make_uint4(0, 0, 0, 0);
    if (g < nfull) {
      a = wc::ld_nc_v4(src + 16 * g);
      bq = wc::ld_nc_v4(src + 16 * g + 8);
      nibbles4(slots4(lut, a.x, a.y), missed);
      nibbles4(slots4(lut, a.z, a.w), missed);
      nibbles4(slots4(lut, bq.x, bq.y), missed);
      nibbles4(slots4(lut, bq.z, bq.w), missed);
    } else if (g == nfull && tail) {
      for (uint32_t j = 0; j < tail; j++) missed += lut[src[16 * g + j] >> 8] == 0xFFu ? 1u : 0u;
    }
    uint32_t total;
    uint64_t e = e0 + r + warp_excl_scan(missed, total);
    for_misses(lut, src, g, nfull, tail, a, bq, missed, [&](uint32_t p, uint32_t h) {
      exc_pos[e] = uint16_t(p);
      exc_val[e] = uint8_t(h);
      e++;
    });
    r += total;
  }
}

__global__ void __launch_bounds__(kPackThreads) k12_pack(const __grid_constant__ EncBatch12 b) {
  __shared__ uint8_t lut[256];
  __shared__ uint32_t staged[kPackWarps][kStaged];  // position | high byte << 16
  __shared__ uint32_t wcount[kPackWarps];
  const EncItem12 &it =
      b.items[find_item(b.items, b.count, blockIdx.x, [](const EncItem12 &x) { return x.chunk_base; })];
  const uint16_t *__restrict__ in = it.in;
  const uint64_t n = it.n;
  uint8_t *out = it.out;
  const uint8_t *scr = it.scr;
  const int tid = threadIdx.x;
  const uint32_t w = uint32_t(tid) >> 5, lane = uint32_t(tid) & 31u;
  lut[tid] = scr[kScrLut + tid];
  const uint64_t c = blockIdx.x - it.chunk_base, v0 = c * kChunk;
  const uint32_t count = uint32_t(n - v0 < kChunk ? n - v0 : kChunk);
  const uint32_t nfull = count / 16, tail = count % 16;
  const uint32_t ngroups = nfull + (tail ? 1u : 0u);
  const uint64_t *h64 = reinterpret_cast<const uint64_t *>(out);
  const uint64_t ne = h64[3];
  const Lay L = lay(n, ne);
  const uint64_t e_base = reinterpret_cast<const uint64_t *>(out + kExcOffOff)[c];
  uint16_t *exc_pos = reinterpret_cast<uint16_t *>(out + L.off_exc);
  uint8_t *exc_val = out + L.off_excval;
  uint8_t *idx_plane = out + L.off_idx + v0 / 2;
  uint8_t *lo_plane = out + L.off_lo + v0;
  const uint16_t *src = in + v0;
  const uint32_t g0 = w * kWarpGroups;
  const uint32_t g1 = g0 + kWarpGroups < ngroups ? g0 + kWarpGroups : ngroups;
  __syncthreads();

  uint32_t wrun = 0;  // this warp's exceptions so far
  // each step's groups are loaded during the step before
  uint4 na = make_uint4(0, 0, 0, 0), nb = make_uint4(0, 0, 0, 0);
  if (g0 + lane < nfull) {
    na = wc::ld_nc_v4(src + 16 * (g0 + lane));
    nb = wc::ld_nc_v4(src + 16 * (g0 + lane) + 8);
  }
  for (uint32_t gs = g0; gs < g1; gs += 32) {
    const uint32_t g = gs + lane;
    uint32_t missed = 0;
    const uint4 a = na, bq = nb;
    if (gs + 32 < g1 && g + 32 < nfull) {
      na = wc::ld_nc_v4(src + 16 * (g + 32));
      nb = wc::ld_nc_v4(src + 16 * (g + 32) + 8);
    }
    if (g < nfull) {
      const uint32_t q0 = nibbles4(slots4(lut, a.x, a.y), missed);
      const uint32_t q1 = nibbles4(slots4(lut, a.z, a.w), missed);
      const uint32_t q2 = nibbles4(slots4(lut, bq.x, bq.y), missed);
      const uint32_t q3 = nibbles4(slots4(lut, bq.z, bq.w), missed);
      *reinterpret_cast<uint2 *>(idx_plane + 8 * g) = make_uint2(q0 | (q1 << 16), q2 | (q3 << 16));
      *reinterpret_cast<uint4 *>(lo_plane + 16 * g) =
          make_uint4(__byte_perm(a.x, a.y, 0x6420), __byte_perm(a.z, a.w, 0x6420),
                     __byte_perm(bq.x, bq.y, 0x6420), __byte_perm(bq.z, bq.w, 0x6420));
    } else if (g == nfull && tail) {
      uint32_t pair = 0;
      for (uint32_t j = 0; j < tail; j++) {
        const uint32_t v = src[16 * g + j];
        const uint32_t s = lut[v >> 8];
        const uint32_t nib = s == 0xFFu ? 0u : s;
        missed += s == 0xFFu ? 1u : 0u;
        pair |= nib << (4 * (j & 1));
        if (j & 1) {
          idx_plane[8 * g + j / 2] = uint8_t(pair);
          pair = 0;
        }
        lo_plane[16 * g + j] = uint8_t(v & 0xFFu);
      }
      if (tail & 1) idx_plane[8 * g + tail / 2] = uint8_t(pair);  // high nibble 0
    }
    // this step's exceptions, in lane order, staged while there is room
    if (__any_sync(0xffffffffu, missed != 0)) {
      uint32_t total;
      uint32_t pos = wrun + warp_excl_scan(missed, total);
      for_misses(lut, src, g, nfull, tail, a, bq, missed, [&](uint32_t p, uint32_t h) {
        if (pos < kStaged) staged[w][pos] = p | (h << 16);
        pos++;
      });
      wrun += total;
    }
  }
  if (lane == 0) wcount[w] = wrun;
  __syncthreads();
  uint64_t e0 = e_base;
  for (uint32_t q = 0; q < w; q++) e0 += wcount[q];
  if (wrun <= kStaged) {
    for (uint32_t i = lane; i < wrun; i += 32) {
      const uint32_t v = staged[w][i];
      exc_pos[e0 + i] = uint16_t(v);
      exc_val[e0 + i] = uint8_t(v >> 16);
    }
  } else {
    rewrite_misses(lut, src, g0, g1, nfull, tail, e0, exc_pos, exc_val);
  }
}

// ---------------------------------------------------------------------------
constexpr int kDecThreads = 256;

// any of the 8 nibbles of w at or above k (1 <= k <= 16)
__device__ __forceinline__ uint32_t over8(uint32_t w, uint32_t add) {
  const uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;
  return ((e + add) | (o + add)) & 0x10101010u;
}

// A container's header and layout, checked (every block that decodes from
// it checks them; the first reports): err is WC_OK, WC_ERR_CORRUPT or, when
// its values do not fit out_cap bytes, WC_ERR_CAPACITY.
struct View12 {
  int32_t err;
  uint64_t n, ne;
  uint32_t k;
  Lay L;
};

__device__ View12 view12(const uint8_t *cont, uint64_t cont_bytes, uint64_t out_cap) {
  View12 v{};
  v.err = WC_ERR_CORRUPT;
  if (cont_bytes < 96) return v;
  const uint32_t *h32 = reinterpret_cast<const uint32_t *>(cont);
  const uint64_t *h64 = reinterpret_cast<const uint64_t *>(cont);
  const uint64_t n = h64[1], ne = h64[3];
  const uint32_t k = h32[1] >> 24;
  bool ok = h32[0] == kMagic && (h32[1] & 0xFFFFFFu) == (1u | (1u << 16)) && k <= 16 &&
            (n > 0) == (k > 0) && n <= kMaxN && ne <= n && h32[4] == uint32_t(kChunk);
  if (!ok) return v;
  const Lay L = lay(n, ne);
  ok = h32[5] == uint32_t(L.nc) && h64[4] == L.off_idx && h64[5] == L.off_lo && h64[6] == L.off_exc &&
       h64[7] == L.total && L.total <= cont_bytes;
  if (!ok) return v;
  // an empty tensor's table is one zero
  if (L.nc == 0 && reinterpret_cast<const uint64_t *>(cont + kExcOffOff)[0] != 0) return v;
  v.n = n;
  v.ne = ne;
  v.k = k;
  v.L = L;
  v.err = 2 * n > out_cap ? WC_ERR_CAPACITY : WC_OK;
  return v;
}

// Chunk c of a checked container into out (whole block): 16 values per
// thread per step, then the chunk's exceptions after a block barrier.
__device__ __forceinline__ void decode_chunk12(const uint8_t *__restrict__ cont, const View12 &v, uint64_t c,
                                               uint16_t *__restrict__ out, int32_t *status) {
  const int tid = threadIdx.x;
  const Lay &L = v.L;
  const uint64_t n = v.n, ne = v.ne;
  const uint32_t k = v.k;
  const uint4 book = *reinterpret_cast<const uint4 *>(cont + kBookOff);
  const uint32_t add = (16u - k) * 0x01010101u;
  const uint64_t *exc_off = reinterpret_cast<const uint64_t *>(cont + kExcOffOff);
  const uint16_t *exc_pos = reinterpret_cast<const uint16_t *>(cont + L.off_exc);
  const uint8_t *exc_val = cont + L.off_excval;
  const uint8_t *idx_plane = cont + L.off_idx;
  const uint8_t *lo_plane = cont + L.off_lo;
  const uint64_t e0 = exc_off[c], e1 = exc_off[c + 1];
  if (!(e0 <= e1 && e1 <= ne && (c != 0 || e0 == 0) && (c + 1 != L.nc || e1 == ne))) {
    if (tid == 0) report(status, WC_ERR_CORRUPT);
    return;
  }
  const uint64_t v0 = c * kChunk;
  const uint32_t count = uint32_t(n - v0 < kChunk ? n - v0 : kChunk);
  const uint32_t nfull = count / 16, tail = count % 16;
  uint32_t bad = 0;
  // U groups a thread with their loads in flight together (plain stores:
  // the streaming hint measured slower here)
  constexpr uint32_t U = 4;
  uint32_t g = tid;
  for (; g + (U - 1) * kDecThreads < nfull; g += U * kDecThreads) {
    uint2 q[U];
    uint4 lo[U];
#pragma unroll
    for (uint32_t u = 0; u < U; u++) {
      const uint32_t gu = g + u * kDecThreads;
      q[u] = __ldg(reinterpret_cast<const uint2 *>(idx_plane + v0 / 2 + 8 * gu));
      lo[u] = __ldg(reinterpret_cast<const uint4 *>(lo_plane + v0 + 16 * gu));
    }
#pragma unroll
    for (uint32_t u = 0; u < U; u++) {
      const uint32_t gu = g + u * kDecThreads;
      bad |= over8(q[u].x, add) | over8(q[u].y, add);
      const uint2 o0 = expand4(q[u].x, book, lo[u].x), o1 = expand4(q[u].x >> 16, book, lo[u].y);
      const uint2 o2 = expand4(q[u].y, book, lo[u].z), o3 = expand4(q[u].y >> 16, book, lo[u].w);
      uint4 *dst = reinterpret_cast<uint4 *>(out + v0 + 16 * gu);
      dst[0] = make_uint4(o0.x, o0.y, o1.x, o1.y);
      dst[1] = make_uint4(o2.x, o2.y, o3.x, o3.y);
    }
  }
  for (; g < nfull; g += kDecThreads) {
    const uint2 q = *reinterpret_cast<const uint2 *>(idx_plane + v0 / 2 + 8 * g);
    const uint4 lo = *reinterpret_cast<const uint4 *>(lo_plane + v0 + 16 * g);
    bad |= over8(q.x, add) | over8(q.y, add);
    const uint2 o0 = expand4(q.x, book, lo.x), o1 = expand4(q.x >> 16, book, lo.y);
    const uint2 o2 = expand4(q.y, book, lo.z), o3 = expand4(q.y >> 16, book, lo.w);
    uint4 *dst = reinterpret_cast<uint4 *>(out + v0 + 16 * g);
    dst[0] = make_uint4(o0.x, o0.y, o1.x, o1.y);
    dst[1] = make_uint4(o2.x, o2.y, o3.x, o3.y);
  }
  if (tid == 0) {  // the ragged tail, value by value
    for (uint32_t j = 0; j < tail; j++) {
      const uint64_t vv = v0 + 16 * uint64_t(nfull) + j;
      const uint32_t nib = (uint32_t(idx_plane[vv / 2]) >> (4 * (vv & 1))) & 0xFu;
      bad |= nib >= k ? 1u : 0u;
      const uint32_t hi = (nib < 8 ? ((&book.x)[nib >> 2] >> (8 * (nib & 3)))
                                   : ((&book.z)[(nib - 8) >> 2] >> (8 * (nib & 3)))) & 0xFFu;
      out[vv] = uint16_t((hi << 8) | lo_plane[vv]);
    }
  }
  if (bad) report(status, WC_ERR_CORRUPT);
  __syncthreads();  // the chunk's values are written; patch its exceptions
  for (uint64_t e = e0 + tid; e < e1; e += kDecThreads) {
    const uint32_t p = exc_pos[e];
    if (p >= count || (e > e0 && p <= exc_pos[e - 1])) {
      report(status, WC_ERR_CORRUPT);
      continue;
    }
    const uint64_t vv = v0 + p;
    out[vv] = uint16_t((uint32_t(exc_val[e]) << 8) | lo_plane[vv]);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kDecThreads)
k12_decode(const uint8_t *__restrict__ cont, uint64_t cont_bytes, uint16_t *__restrict__ out,
           uint64_t out_cap, int32_t *status) {
  const View12 v = view12(cont, cont_bytes, out_cap);
  if (v.err != WC_OK) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, v.err);
    return;
  }
  for (uint64_t c = blockIdx.x; c < v.L.nc; c += gridDim.x) decode_chunk12(cont, v, c, out, status);
}

// Many containers in one launch: work unit g (a chunk, or the one unit of an
// empty tensor) of the container whose units start at or before g.
__global__ void __launch_bounds__(kDecThreads) k12_decode_batch(const __grid_constant__ DecBatch12 b) {
  for (uint32_t g = blockIdx.x; g < b.total_units; g += gridDim.x) {
    const DecItem12 &it =
        b.items[find_item(b.items, b.count, g, [](const DecItem12 &x) { return x.unit_base; })];
    const uint32_t u = g - it.unit_base;
    const View12 v = view12(it.cont, it.cont_bytes, 2 * it.n);
    // a header for another number of values is not the tensor the caller expects
    const int32_t err = v.err != WC_ERR_CORRUPT && v.n != it.n ? WC_ERR_CORRUPT : v.err;
    if (err != WC_OK) {
      if (u == 0 && threadIdx.x == 0) report(b.status, err);
      continue;
    }
    if (v.L.nc > 0) decode_chunk12(it.cont, v, u, it.out, b.status);
  }
}

int sms_of_current_device() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = sms;
  }
  return cache[dev];
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace wc12

extern "C" {

uint64_t wc12_encode_bound(uint64_t n) {
  if (n > wc12::kMaxN) return 0;
  return wc12::lay(n, n - (n + 15) / 16).total;
}

uint64_t wc12_scratch_bytes(uint64_t n) {
  if (n > wc12::kMaxN) return 0;
  return wc12::kScrChunkHist + 1024 * ((n + wc12::kChunk - 1) / wc12::kChunk);
}

int32_t wc12_encode_batch(const wc12_encode_item *items, uint32_t count, void *stream) {
  if (count == 0) return WC_OK;
  if (items == nullptr) return WC_ERR_INVALID_ARG;
  for (uint32_t i = 0; i < count; i++) {
    const wc12_encode_item &it = items[i];
    if (it.n > wc12::kMaxN || it.out == nullptr || it.scratch == nullptr || it.out_size == nullptr)
      return WC_ERR_INVALID_ARG;
    if (it.n > 0 && it.in == nullptr) return WC_ERR_INVALID_ARG;
    if (!wc12::aligned(it.in, 16) || !wc12::aligned(it.out, 16) || !wc12::aligned(it.scratch, 16) ||
        !wc12::aligned(it.out_size, 8))
      return WC_ERR_INVALID_ARG;
    if (it.out_cap < wc12_encode_bound(it.n) || it.scratch_cap < wc12_scratch_bytes(it.n)) return WC_ERR_CAPACITY;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local wc12::EncBatch12 B;  // ~12 KiB: kept off the stack
  for (uint32_t b0 = 0; b0 < count; b0 += wc12::kBatchMax) {
    const uint32_t cnt = count - b0 < wc12::kBatchMax ? count - b0 : wc12::kBatchMax;
    memset(&B, 0, sizeof(B));
    B.count = cnt;
    uint64_t chunks = 0, cblocks = 0;
    for (uint32_t i = 0; i < cnt; i++) {
      const wc12_encode_item &src = items[b0 + i];
      wc12::EncItem12 &d = B.items[i];
      d.in = static_cast<const uint16_t *>(src.in);
      d.out = static_cast<uint8_t *>(src.out);
      d.scr = static_cast<uint8_t *>(src.scratch);
      d.out_size = src.out_size;
      d.n = src.n;
      d.chunk_base = uint32_t(chunks);
      d.count_base = uint32_t(cblocks);
      const uint64_t nc = (src.n + wc12::kChunk - 1) / wc12::kChunk;
      chunks += nc;
      cblocks += nc ? (nc + 7) / 8 : 1;  // an empty tensor's block writes exc_off[0]
      if (chunks > 0x7FFFFFFFull || cblocks > 0x7FFFFFFFull) return WC_ERR_INVALID_ARG;
    }
    B.total_chunks = uint32_t(chunks);
    B.total_count_blocks = uint32_t(cblocks);
    wc12::k12_prep<<<cnt, 256, 0, s>>>(B);
    if (chunks) wc12::k12_hist<<<unsigned(chunks), wc12::kHistThreads, 0, s>>>(B);
    wc12::k12_book<<<cnt, 256, 0, s>>>(B);
    wc12::k12_count<<<unsigned(cblocks), 256, 0, s>>>(B);
    wc12::k12_scan<<<cnt, wc12::kScanThreads, 0, s>>>(B);
    if (chunks) wc12::k12_pack<<<unsigned(chunks), wc12::kPackThreads, 0, s>>>(B);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
  }
  return WC_OK;
}

int32_t wc12_encode(const void *d_in, uint64_t n, void *d_out, uint64_t out_cap, void *d_scratch,
                    uint64_t scratch_cap, uint64_t *d_out_size, void *stream) {
  wc12_encode_item it{d_in, n, d_out, out_cap, d_scratch, scratch_cap, d_out_size};
  return wc12_encode_batch(&it, 1, stream);
}

int32_t wc12_read_header(const void *h_cont, uint64_t bytes, uint64_t *n, uint64_t *ne, uint32_t *k) {
  if (h_cont == nullptr || n == nullptr || ne == nullptr || k == nullptr) return WC_ERR_INVALID_ARG;
  if (bytes < 96) return WC_ERR_CORRUPT;
  uint32_t h32[16];
  memcpy(h32, h_cont, 64);
  uint64_t h64[8];
  memcpy(h64, h_cont, 64);
  const uint64_t nn = h64[1], nne = h64[3];
  const uint32_t kk = h32[1] >> 24;
  if (h32[0] != wc12::kMagic || (h32[1] & 0xFFFFFFu) != (1u | (1u << 16)) || kk > 16 ||
      (nn > 0) != (kk > 0) || nn > wc12::kMaxN || nne > nn || h32[4] != uint32_t(wc12::kChunk))
    return WC_ERR_CORRUPT;
  const wc12::Lay L = wc12::lay(nn, nne);
  if (h32[5] != uint32_t(L.nc) || h64[4] != L.off_idx || h64[5] != L.off_lo || h64[6] != L.off_exc ||
      h64[7] != L.total || L.total > bytes)
    return WC_ERR_CORRUPT;
  *n = nn;
  *ne = nne;
  *k = kk;
  return WC_OK;
}

int32_t wc12_decode_batch(const wc12_decode_item *items, uint32_t count, int32_t *d_status, void *stream) {
  if (count == 0) return WC_OK;
  if (items == nullptr || d_status == nullptr || !wc12::aligned(d_status, 4)) return WC_ERR_INVALID_ARG;
  for (uint32_t i = 0; i < count; i++) {
    const wc12_decode_item &it = items[i];
    if (it.cont == nullptr || !wc12::aligned(it.cont, 16) || !wc12::aligned(it.out, 16) || it.n > wc12::kMaxN)
      return WC_ERR_INVALID_ARG;
    if (it.n > 0 && it.out == nullptr) return WC_ERR_INVALID_ARG;
  }
  const int sms = wc12::sms_of_current_device();
  if (sms <= 0) return WC_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local wc12::DecBatch12 B;
  for (uint32_t b0 = 0; b0 < count; b0 += wc12::kBatchMax) {
    const uint32_t cnt = count - b0 < wc12::kBatchMax ? count - b0 : wc12::kBatchMax;
    memset(&B, 0, sizeof(B));
    B.count = cnt;
    B.status = d_status;
    uint64_t units = 0;
    for (uint32_t i = 0; i < cnt; i++) {
      const wc12_decode_item &src = items[b0 + i];
      wc12::DecItem12 &d = B.items[i];
      d.cont = static_cast<const uint8_t *>(src.cont);
      d.cont_bytes = src.cont_bytes;
      d.out = static_cast<uint16_t *>(src.out);
      d.n = src.n;
      d.unit_base = uint32_t(units);
      const uint64_t nc = (src.n + wc12::kChunk - 1) / wc12::kChunk;
      units += nc ? nc : 1;
      if (units > 0x7FFFFFFFull) return WC_ERR_INVALID_ARG;
    }
    B.total_units = uint32_t(units);
    // one block per unit: the hardware hands the next unit to whichever block
    // slot frees first (a fixed share per block of a persistent grid left
    // the faster blocks of an SM idle while its slower ones finished)
    wc12::k12_decode_batch<<<unsigned(units), wc12::kDecThreads, 0, s>>>(B);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
  }
  return WC_OK;
}

int32_t wc12_decode(const void *d_cont, uint64_t cont_bytes, void *d_out, uint64_t out_cap,
                    int32_t *d_status, void *stream) {
  if (d_cont == nullptr || d_status == nullptr) return WC_ERR_INVALID_ARG;
  if (!wc12::aligned(d_cont, 16) || !wc12::aligned(d_out, 16) || !wc12::aligned(d_status, 4))
    return WC_ERR_INVALID_ARG;
  if (out_cap > 0 && d_out == nullptr) return WC_ERR_INVALID_ARG;
  const int sms = wc12::sms_of_current_device();
  if (sms <= 0) return WC_ERR_CUDA;
  // one block per chunk the output can hold (the header, read on the device,
  // gives the count; blocks past it have nothing to do)
  uint64_t blocks = (out_cap / 2 + wc12::kChunk - 1) / wc12::kChunk;
  if (blocks < 1) blocks = 1;
  if (blocks > (uint64_t(1) << 24)) blocks = uint64_t(1) << 24;
  wc12::k12_decode<<<unsigned(blocks), wc12::kDecThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t *>(d_cont), cont_bytes, static_cast<uint16_t *>(d_out), out_cap,
      d_status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return WC_ERR_CUDA;
  return WC_OK;
}

}  // extern "C"
