// wc_format.cuh -- container constants, section layout and kernel launch
// parameters shared by the CUDA kernels and the host entry points of the
// exponent-plane rANS codec.  (The CPU oracle restates all of this on its
// own; nothing here is shared with it.)
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "wc.h"

namespace wc {

// Container parameters: 65,536-symbol chunks, 32 interleaved lanes, 12-bit
// static table (sum 4096), 32-bit states in [2^16, 2^32), 16-bit words.
constexpr uint32_t kChunk = 65536;
constexpr uint32_t kLanes = 32;
constexpr uint32_t kProbBits = 12;
constexpr uint32_t kProbScale = 1u << kProbBits;  // M = 4096
constexpr uint32_t kStateLow = 1u << 16;          // L = 2^16
constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kFreqOffset = 64;
constexpr uint32_t kChunkOffOffset = 576;  // 64 + 2 * 256
constexpr uint32_t kStateBytes = kLanes * 4;  // 128
constexpr uint32_t kVersion = 1;

// Each lane handles 16 consecutive values per "group" of 16 steps: one group
// is 512 values, 128 groups make a full chunk.
constexpr uint32_t kGroupValues = 512;
constexpr uint32_t kStepsPerGroup = 16;

// Encoder scratch, per tensor (offsets in bytes from the tensor's scratch).
//   hist     u64[256]       coded-byte counts
//   ctr      u32[4]         [0] histogram blocks done, [1] coder warps done,
//                           [2] table written: 1 narrow, 2 wide format, [3] unused
//   tab      uint4[256]     per-symbol coding entry (wc_coder.cuh): narrow {m,
//                           xmax, cmpl, sh | bias << 5}, wide {ml, xmax, cmpl, mh}
//   bias     u32[256]       per-symbol additive term (wide format)
//   len      u32[nc]        chunk lengths
//   windows  nc x kWin      coded chunk staging (states at the front,
//                           words filled backwards from the end)
constexpr uint64_t kScrHist = 0;
constexpr uint64_t kScrCtr = 2048;
constexpr uint64_t kScrTab = 2304;
constexpr uint64_t kScrBias = kScrTab + 256 * 16;   // 6400
constexpr uint64_t kScrLen = kScrBias + 256 * 4;    // 7424
constexpr uint64_t kWin = 65536 + 2048;             // 67584 bytes per chunk
constexpr uint32_t kWinWords = kWin / 2;            // 33792

// fp8 e4m3 and e5m2: one byte per value, the raw plane one nibble per value.
__host__ __device__ constexpr bool is_fp8(int dt) { return dt == WC_FP8E4M3 || dt == WC_FP8E5M2; }

__host__ __device__ inline uint64_t round16(uint64_t v) { return (v + 15) & ~uint64_t(15); }
__host__ __device__ inline uint64_t round256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

__host__ __device__ inline uint64_t num_chunks(uint64_t n) { return (n + kChunk - 1) / kChunk; }

__host__ __device__ inline uint32_t chunk_nsym(uint64_t n, uint64_t k) {
  uint64_t left = n - k * kChunk;
  return left < kChunk ? uint32_t(left) : kChunk;
}

struct Layout {
  uint64_t n, nc;
  uint64_t off_chunk_off, off_chunk_len;
  uint64_t off_raw;   // bf16: sign+mantissa bytes; fp16: low bytes; fp8: low nibbles; fp32: sign bits
  uint64_t off_mant;  // fp32 only
  uint64_t off_exp;
};

__host__ __device__ inline Layout make_layout(uint64_t n, int dtype) {
  Layout L;
  L.n = n;
  L.nc = num_chunks(n);
  L.off_chunk_off = kChunkOffOffset;
  L.off_chunk_len = L.off_chunk_off + 8 * (L.nc + 1);
  L.off_raw = round16(L.off_chunk_len + 4 * L.nc);
  if (dtype == WC_BF16 || dtype == WC_FP16) {  // one raw byte per value
    L.off_mant = 0;
    L.off_exp = round16(L.off_raw + n);
  } else if (is_fp8(dtype)) {  // one raw nibble per value
    L.off_mant = 0;
    L.off_exp = round16(L.off_raw + (n + 1) / 2);
  } else {
    L.off_mant = round16(L.off_raw + (n + 7) / 8);
    L.off_exp = round16(L.off_mant + 3 * n);
  }
  return L;
}

// Bytes per value.
__host__ __device__ constexpr uint32_t dtype_bytes(int dtype) {
  return dtype == WC_FP32 ? 4 : (is_fp8(dtype) ? 1 : 2);
}

__host__ __device__ inline uint64_t scratch_win_offset(uint64_t nc) {
  return round256(kScrLen + 4 * nc);
}

// ---------------------------------------------------------------------------
// Launch parameters (passed by value; up to kMaxItems tensors per launch).
// ---------------------------------------------------------------------------
constexpr uint32_t kMaxItems = 256;

struct EncItem {
  const uint8_t *in;
  uint8_t *out;
  uint8_t *scratch;
  uint64_t *out_size;
  uint64_t n;
  uint32_t chunk_base;  // first global chunk index of this item in the launch
  uint32_t block_base;  // first coder block of this item in the launch
  uint32_t dtype;
  uint32_t hist_base;   // first histogram block of this item in the launch
};

struct EncParams {
  uint32_t count;
  uint32_t total_chunks;
  uint32_t total_coder_blocks;
  uint32_t total_hist_blocks;
  EncItem items[kMaxItems];
};

struct DecItem {
  const uint8_t *cont;
  uint64_t cont_bytes;
  uint8_t *out;
  uint64_t out_cap;
  uint64_t chunk_first;  // first chunk decoded
  uint64_t chunk_count;  // UINT64_MAX: through the last chunk
};

struct DecParams {
  uint32_t count;
  uint32_t pad[3];
  int32_t *status;
  uint32_t *queue;  // this launch's counter of groups taken (set by launch_decode)
  DecItem items[kMaxItems];
};

// Histogram blocks: one tile of up to 4 chunks of one tensor.
constexpr uint32_t kHistChunks = 4;
// Encoder coder blocks: 8 warps, two chunks each, all of one tensor.
constexpr uint32_t kCoderWarps = 8;
constexpr uint32_t kCoderChunks = 2 * kCoderWarps;
// Decoder blocks: 8 warps, two chunks each, all of one tensor.
constexpr uint32_t kDecWarps = 8;

// Host launchers (one per kernel file).
cudaError_t launch_prep(const EncParams &p, cudaStream_t s);
cudaError_t launch_hist(const EncParams &p, cudaStream_t s);
cudaError_t launch_coder(const EncParams &p, cudaStream_t s);
cudaError_t launch_compact(const EncParams &p, cudaStream_t s);
cudaError_t launch_decode(DecParams &p, int grid, cudaStream_t s);
int decode_blocks_per_sm();
// Identity of the CUDA context current on this thread, 0 if none (for
// caching device addresses of the library's own device arrays).
unsigned long long current_context_id();

// ---------------------------------------------------------------------------
// Device helpers.
// ---------------------------------------------------------------------------
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t find_item_by_chunk(const EncParams &p, uint32_t g) {
  uint32_t lo = 0, hi = p.count - 1;
  while (lo < hi) {
    uint32_t mid = (lo + hi + 1) >> 1;
    if (p.items[mid].chunk_base <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint32_t find_item_by_block(const EncParams &p, uint32_t b) {
  uint32_t lo = 0, hi = p.count - 1;
  while (lo < hi) {
    uint32_t mid = (lo + hi + 1) >> 1;
    if (p.items[mid].block_base <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint32_t find_item_by_hist(const EncParams &p, uint32_t b) {
  uint32_t lo = 0, hi = p.count - 1;
  while (lo < hi) {
    uint32_t mid = (lo + hi + 1) >> 1;
    if (p.items[mid].hist_base <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}
#endif

}  // namespace wc
