// wc_planes.cuh -- the two byte planes of a 2-byte value and back ("PTWM",
// How it works 1-2: the reorder S E M -> E S M, then the value is cut into its
// bytes and the high, exponent-bearing byte is the one that is coded).
//   bf16 [S:1 E:8 M:7]   coded byte E                       raw byte S<<7 | M
//   fp16 [S:1 E:5 M:10]  coded byte E<<3 | S<<2 | M>>8      raw byte M & 0xFF
// The scalar forms take one 16-bit value.  The x4 forms work on four values
// at once, one per byte lane: w0 = [v1:v0] and w1 = [v3:v2] are the values as
// two 32-bit words; c4 / r4 hold the four coded / raw bytes, value j in byte j.
#pragma once

#include <cstdint>

#include "wc.h"
#include "wc_format.cuh"

namespace wc {

template <int DT>
__device__ __forceinline__ uint32_t code_byte(uint32_t v) {
  if (DT == WC_BF16) return (v >> 7) & 0xFFu;
  return ((v >> 7) & 0xF8u) | ((v >> 13) & 0x04u) | ((v >> 8) & 0x03u);
}

template <int DT>
__device__ __forceinline__ uint32_t raw_byte(uint32_t v) {
  if (DT == WC_BF16) return ((v >> 8) & 0x80u) | (v & 0x7Fu);
  return v & 0xFFu;
}

template <int DT>
__device__ __forceinline__ uint32_t merge16(uint32_t code, uint32_t raw) {
  if (DT == WC_BF16) return ((raw & 0x80u) << 8) | (code << 7) | (raw & 0x7Fu);
  const uint32_t hi = ((code >> 1) & 0x7Cu) | ((code << 5) & 0x80u) | (code & 0x03u);
  return (hi << 8) | raw;
}

template <int DT>
__device__ __forceinline__ uint32_t code4(uint32_t w0, uint32_t w1) {
  if (DT == WC_BF16) return __byte_perm(w0 >> 7, w1 >> 7, 0x6420);
  const uint32_t hb = __byte_perm(w0, w1, 0x7531);  // the four high bytes
  return ((hb << 1) & 0xF8F8F8F8u) | ((hb >> 5) & 0x04040404u) | (hb & 0x03030303u);
}

template <int DT>
__device__ __forceinline__ uint32_t raw4(uint32_t w0, uint32_t w1) {
  const uint32_t lo = __byte_perm(w0, w1, 0x6420);  // the four low bytes
  if (DT == WC_BF16) {
    const uint32_t hi = __byte_perm(w0, w1, 0x7531);
    return (lo & 0x7F7F7F7Fu) | (hi & 0x80808080u);
  }
  return lo;
}

template <int DT>
__device__ __forceinline__ uint2 merge4(uint32_t c4, uint32_t r4) {
  uint32_t lo, hi;  // the four values' low and high bytes
  if (DT == WC_BF16) {
    lo = (r4 & 0x7F7F7F7Fu) | ((c4 << 7) & 0x80808080u);
    hi = ((c4 >> 1) & 0x7F7F7F7Fu) | (r4 & 0x80808080u);
  } else {
    lo = r4;
    hi = ((c4 >> 1) & 0x7C7C7C7Cu) | ((c4 << 5) & 0x80808080u) | (c4 & 0x03030303u);
  }
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// ---------------------------------------------------------------------------
// fp8, one byte per value.  e4m3 [S:1 E:4 M:3]: the reorder gives
// E<<4 | S<<3 | M, so the coded symbol is the exponent nibble E and the raw
// nibble is S<<3 | M.  e5m2 [S:1 E:5 M:2]: the reorder gives E<<3 | S<<2 | M,
// the coded symbol is the high nibble, exponent bits 4..1, and the raw nibble
// is E0<<3 | S<<2 | M ("PTWM" How it works 1-2: the exponent goes to the high
// nibble, then the byte is cut into nibbles).  Both codes are bits 6..3 of
// the value.  Raw nibbles are stored two per byte, even value in the low
// half.  The x4 / x8 forms work on four values per 32-bit word, one per byte
// lane.

__device__ __forceinline__ uint32_t fp8_code(uint32_t b) { return (b >> 3) & 0xFu; }
template <int DT>
__device__ __forceinline__ uint32_t fp8_nibble(uint32_t b) {
  if (DT == WC_FP8E4M3) return ((b >> 4) & 8u) | (b & 7u);
  return ((b << 1) & 8u) | ((b >> 5) & 4u) | (b & 3u);
}
template <int DT>
__device__ __forceinline__ uint32_t fp8_merge(uint32_t code, uint32_t nib) {
  if (DT == WC_FP8E4M3) return ((nib & 8u) << 4) | ((code & 0xFu) << 3) | (nib & 7u);
  return ((nib & 4u) << 5) | ((code & 0xFu) << 3) | ((nib & 8u) >> 1) | (nib & 3u);
}

__device__ __forceinline__ uint32_t fp8_code4(uint32_t w) { return (w >> 3) & 0x0F0F0F0Fu; }
template <int DT>
__device__ __forceinline__ uint32_t fp8_nibble4(uint32_t w) {
  if (DT == WC_FP8E4M3) return ((w >> 4) & 0x08080808u) | (w & 0x07070707u);
  return ((w << 1) & 0x08080808u) | ((w >> 5) & 0x04040404u) | (w & 0x03030303u);
}
// the low nibbles of 8 values (two words) packed into 4 bytes
template <int DT>
__device__ __forceinline__ uint32_t fp8_pack8(uint32_t w0, uint32_t w1) {
  const uint32_t t0 = fp8_nibble4<DT>(w0), t1 = fp8_nibble4<DT>(w1);
  return __byte_perm(t0 | (t0 >> 4), t1 | (t1 >> 4), 0x6420);
}
// four values from four codes (c4) and four nibbles (n4), one per byte lane
template <int DT>
__device__ __forceinline__ uint32_t fp8_merge4(uint32_t c4, uint32_t n4) {
  if (DT == WC_FP8E4M3)
    return ((n4 & 0x08080808u) << 4) | ((c4 & 0x0F0F0F0Fu) << 3) | (n4 & 0x07070707u);
  return ((n4 & 0x04040404u) << 5) | ((c4 & 0x0F0F0F0Fu) << 3) | ((n4 & 0x08080808u) >> 1) |
         (n4 & 0x03030303u);
}
// 8 values (coded bytes c8, packed nibbles r) -> 8 value bytes as two words
template <int DT>
__device__ __forceinline__ uint2 fp8_merge8(uint2 c8, uint32_t r) {
  const uint32_t lo = r & 0x0F0F0F0Fu, hi = (r >> 4) & 0x0F0F0F0Fu;
  const uint32_t n0 = __byte_perm(lo, hi, 0x5140), n1 = __byte_perm(lo, hi, 0x7362);
  return make_uint2(fp8_merge4<DT>(c8.x, n0), fp8_merge4<DT>(c8.y, n1));
}

}  // namespace wc
