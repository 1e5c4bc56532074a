// wc_coder.cuh -- the rANS coding step's division by the symbol frequency,
// and the per-symbol table entry it reads.
//
// Coding a symbol s with frequency f and cumulative frequency cum from a
// renormalised state x (x < f 2^20) gives x' = (x / f) 4096 + x % f + cum
// = x + (x / f)(4096 - f) + cum; only x / f needs a division, and the coder
// computes it exactly with multiplies:
//   narrow format (every f of the tensor <= 2048): q = floor(x m / 2^k) with
//     k = 31 + c, c = ceil(log2 f), m = ceil(2^k / f) < 2^32, computed as
//     umulhi(x, m) >> (c - 1).  With e = m f - 2^k < f, the error term
//     x e / (f 2^k) < f 2^20 f / (f 2^(31 + c)) <= 1 / f when f <= 2^11, so
//     the floor is exact;
//   wide format (some f > 2048): m = ceil(2^64 / f) as two 32-bit halves,
//     q = the high word of x m / 2^32 (two multiply-adds), exact for every
//     x < 2^32.
// In both, f = 1 uses the all-ones multiplier, which yields q = x - 1, repaid
// by bias += 4095.  One format per tensor: the coder is compiled for both.
#pragma once

#include <cstdint>

#include "wc_format.cuh"

namespace wc {

// Table entry of a symbol with frequency ff > 0 (ff = 0: all zero):
// narrow {m, xmax, 4096 - f, shift | bias << 5}; wide {m low, xmax,
// 4096 - f, m high} with the bias returned separately.  xmax = f 2^20 - 1:
// the state is renormalised while it is above xmax.
__host__ __device__ inline void coder_entry(uint32_t ff, uint32_t cum, bool wide, uint4 &e,
                                            uint32_t &bias) {
  e = make_uint4(0, 0, 0, 0);
  bias = 0;
  if (ff == 0) return;
  bias = cum + (ff == 1 ? kProbScale - 1 : 0);
  e.y = uint32_t((uint64_t(ff) << 20) - 1);
  e.z = kProbScale - ff;
  if (wide) {
    const uint64_t m = ff >= 2 ? (~uint64_t(0) / ff + 1) : ~uint64_t(0);
    e.x = uint32_t(m);
    e.w = uint32_t(m >> 32);
  } else {
    uint32_t m = 0xFFFFFFFFu, sh = 0;
    if (ff >= 2) {
      uint32_t c = 0;  // ceil(log2 ff)
      while ((uint32_t(1) << c) < ff) c++;
      m = uint32_t(((uint64_t(1) << (31 + c)) - 1) / ff + 1);
      sh = c - 1;
    }
    e.x = m;
    e.w = sh | (bias << 5);
  }
}

#ifdef __CUDACC__
// x' = (x / f) 4096 + x % f + cum for a renormalised state x < f 2^20, from
// the symbol's table entry (and, in the wide format, its bias).
template <bool W>
__device__ __forceinline__ uint32_t advance(uint32_t x, const uint4 &te, uint32_t bi) {
  if (W) {
    const uint32_t qlo = __umulhi(x, te.x);
    const uint64_t prod = uint64_t(x) * te.w + qlo;
    return x + uint32_t(prod >> 32) * te.z + bi;
  }
  const uint32_t q = __funnelshift_r(__umulhi(x, te.x), 0u, te.w);  // shift = te.w & 31
  return x + q * te.z + (te.w >> 5);
}
#endif

}  // namespace wc
