// wc_split12.cuh -- the Split12 container layout (include/wc_split12.h) and
// the expansion of index nibbles + low bytes into bf16, shared by the codec
// (k_split12.cu) and the fused linear layer (k_split12_linear.cu).
#pragma once

#include <cstdint>

#include "wc.h"
#include "wc_split12.h"

namespace wc12 {

constexpr uint64_t kChunk = 65536;
constexpr uint32_t kBookOff = 64;
constexpr uint32_t kExcOffOff = 80;
constexpr uint32_t kMagic = 0x43323157u;  // "W12C"
constexpr uint64_t kMaxN = uint64_t(1) << 44;

constexpr uint64_t kScrHist = 0;           // u64[256]
constexpr uint64_t kScrLut = 2048;         // u8[256]
constexpr uint64_t kScrChunkHist = 2560;   // u32[nc][256]

__host__ __device__ inline uint64_t r16(uint64_t v) { return (v + 15) & ~uint64_t(15); }

struct Lay {
  uint64_t nc, off_idx, off_lo, off_exc, off_excval, total;
};

__host__ __device__ inline Lay lay(uint64_t n, uint64_t ne) {
  Lay L;
  L.nc = (n + kChunk - 1) / kChunk;
  L.off_idx = r16(kExcOffOff + 8 * (L.nc + 1));
  L.off_lo = r16(L.off_idx + (n + 1) / 2);
  L.off_exc = r16(L.off_lo + n);
  L.off_excval = L.off_exc + r16(2 * ne);
  L.total = L.off_excval + r16(ne);
  return L;
}

// 4 index nibbles (low 16 bits of q), the codebook in four words, 4 low bytes
// -> the 4 bf16 values as two words
__device__ __forceinline__ uint2 expand4(uint32_t q, uint4 book, uint32_t lo4) {
  const uint32_t sel = q & 0x7777u;              // entry within its half
  const uint32_t upper = (q >> 3) & 0x1111u;     // 1: entries 8..15
  const uint32_t r0 = __byte_perm(book.x, book.y, sel);
  const uint32_t r1 = __byte_perm(book.z, book.w, sel);
  const uint32_t m = __byte_perm(0x0000FF00u, 0u, upper);  // 0xFF where upper
  const uint32_t hi4 = (r0 & ~m) | (r1 & m);
  return make_uint2(__byte_perm(lo4, hi4, 0x5140), __byte_perm(lo4, hi4, 0x7362));
}

}  // namespace wc12
