// k_crc.cu -- CRC-32 of fixed-size blocks of a device buffer, the check that
// an archive keeps per block ("seedpack 0.2.0 -> 0.2.2", README: every chunk
// of an archive carries a CRC32).  The code is the zlib / IEEE 802.3 CRC-32:
// generator G of degree 32, bits taken least significant first, register
// preset to all ones, result complemented.
//
// Arithmetic.  A 32-bit register r stands for a polynomial of degree < 32
// with the coefficient of x^k in bit 31-k.  Feeding one zero bit multiplies
// by x modulo G: shift right, xor 0xEDB88320 (G without x^32, in the same bit
// order) when a 1 falls out.  Write raw(M) for the register after message M
// from a zero register; raw is linear in M, and for a concatenation
//     raw(A B) = raw(A) * x^(8|B|) + raw(B)          (mod G, over GF(2)),
// while the CRC proper is  ~( raw(M) + 0xFFFFFFFF * x^(8|M|) ).
//
// Work split.  One CTA (512 threads) per block at a time, grid-strided over
// the blocks; thread t takes the t-th of 512 equal contiguous segments of the
// block (block_bytes / 512 bytes, a multiple of 16), computes raw() of it with
// 4-byte slicing tables, multiplies it by x^(8 * bytes after the segment) and
// the CTA xors the 512 products.  For full blocks the multiplier of each
// thread is the same in every block and is computed once per launch.
//
// Tables.  S_k[b] = raw(byte b followed by k zero bytes), k = 0..3, give one
// 4-byte step:  r ^= w;  r = S_3[r0] ^ S_2[r1] ^ S_1[r2] ^ S_0[r3]  (ri the
// bytes of r, r0 lowest).  Lookups are data-dependent, so the 4 KiB of
// tables are held 32 times over in shared memory, entry (k, b) of lane l at
// word ((k * 256 + b) * 32 + l): every lane reads its own bank.
#include <cstdint>

#include "wc.h"
#include "wc_format.cuh"

namespace wc {
namespace {

constexpr int kCrcThreads = 512;
constexpr uint32_t kGenReversed = 0xEDB88320u;

struct CrcSmem {
  uint32_t rep[4 * 256 * 32];  // lane-replicated slicing tables, 128 KiB
  uint32_t base[4 * 256];      // the tables once
  uint32_t red[kCrcThreads / 32];
};

extern __shared__ __align__(16) uint8_t crc_smem[];

// a * b mod G, both in the register's bit order
__device__ uint32_t gf_mul(uint32_t a, uint32_t b) {
  uint32_t p = 0;
#pragma unroll 8
  for (int i = 0; i < 32; i++) {
    p ^= b & (0u - (a >> 31));
    a <<= 1;
    b = (b >> 1) ^ (kGenReversed & (0u - (b & 1u)));
  }
  return p;
}

// x^(8n) mod G, by squaring
__device__ uint32_t xpow8(uint64_t n) {
  uint32_t r = 0x80000000u, sq = 0x00800000u;  // x^0, x^8
  while (n) {
    if (n & 1u) r = gf_mul(r, sq);
    sq = gf_mul(sq, sq);
    n >>= 1;
  }
  return r;
}

// t = this lane's column of the replicated tables
__device__ __forceinline__ uint32_t step4(uint32_t r, uint32_t w, const uint32_t *t) {
  r ^= w;
  return t[(768u + (r & 0xFFu)) << 5] ^ t[(512u + ((r >> 8) & 0xFFu)) << 5] ^
         t[(256u + ((r >> 16) & 0xFFu)) << 5] ^ t[(r >> 24) << 5];
}

__device__ __forceinline__ uint32_t step16(uint32_t r, uint4 v, const uint32_t *t) {
  r = step4(r, v.x, t);
  r = step4(r, v.y, t);
  r = step4(r, v.z, t);
  return step4(r, v.w, t);
}

// raw() of n bytes at p (p 16-byte aligned)
__device__ uint32_t raw_segment(const uint8_t *p, uint64_t n, const uint32_t *t) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
  const uint64_t n16 = n >> 4, groups = n16 >> 2;
  uint32_t r = 0;
  if (groups) {
    // 64 bytes in registers while the next 64 are on their way
    uint4 c0 = __ldg(q), c1 = __ldg(q + 1), c2 = __ldg(q + 2), c3 = __ldg(q + 3);
    for (uint64_t g = 1; g < groups; g++) {
      const uint4 *qg = q + 4 * g;
      const uint4 d0 = __ldg(qg), d1 = __ldg(qg + 1), d2 = __ldg(qg + 2), d3 = __ldg(qg + 3);
      r = step16(r, c0, t);
      r = step16(r, c1, t);
      r = step16(r, c2, t);
      r = step16(r, c3, t);
      c0 = d0;
      c1 = d1;
      c2 = d2;
      c3 = d3;
    }
    r = step16(r, c0, t);
    r = step16(r, c1, t);
    r = step16(r, c2, t);
    r = step16(r, c3, t);
  }
  for (uint64_t i = groups * 4; i < n16; i++) r = step16(r, __ldg(q + i), t);
  const uint8_t *b = p + (n16 << 4);
  uint32_t rem = uint32_t(n & 15u);
  for (; rem >= 4; rem -= 4, b += 4) r = step4(r, __ldg(reinterpret_cast<const uint32_t *>(b)), t);
  for (; rem; rem--, b++) r = t[((r ^ __ldg(b)) & 0xFFu) << 5] ^ (r >> 8);
  return r;
}

__global__ void __launch_bounds__(kCrcThreads, 1)
k_crc32(const uint8_t *__restrict__ buf, uint64_t bytes, uint64_t block_bytes,
        uint32_t *__restrict__ crc) {
  CrcSmem &s = *reinterpret_cast<CrcSmem *>(crc_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid < 256) {
    uint32_t r = uint32_t(tid);
    for (int i = 0; i < 8; i++) r = (r >> 1) ^ (kGenReversed & (0u - (r & 1u)));
    s.base[tid] = r;
  }
  __syncthreads();
  if (tid < 256) {
    uint32_t r = s.base[tid];
    for (int k = 1; k < 4; k++) {
      r = s.base[r & 0xFFu] ^ (r >> 8);  // one more zero byte
      s.base[k * 256 + tid] = r;
    }
  }
  __syncthreads();
  for (int i = tid; i < 4 * 256 * 32; i += kCrcThreads) s.rep[i] = s.base[i >> 5];
  __syncthreads();

  const uint32_t *t = s.rep + lane;
  const uint64_t nblocks = (bytes + block_bytes - 1) / block_bytes;
  const uint64_t seg = block_bytes / kCrcThreads;
  // full blocks: what follows thread tid's segment, and the preset's image
  const uint32_t mul_full = xpow8(uint64_t(kCrcThreads - 1 - tid) * seg);
  const uint32_t preset_full = gf_mul(0xFFFFFFFFu, xpow8(block_bytes));

  for (uint64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const uint64_t start = blk * block_bytes;
    const uint64_t len = bytes - start < block_bytes ? bytes - start : block_bytes;
    const uint64_t s0 = uint64_t(tid) * seg < len ? uint64_t(tid) * seg : len;
    const uint64_t s1 = s0 + seg < len ? s0 + seg : len;
    const uint32_t r = raw_segment(buf + start + s0, s1 - s0, t);
    uint32_t part = 0;
    if (r != 0) part = gf_mul(r, len == block_bytes ? mul_full : xpow8(len - s1));
#pragma unroll
    for (int o = 16; o; o >>= 1) part ^= __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (lane == 0) s.red[warp] = part;
    __syncthreads();
    if (tid == 0) {
      uint32_t x = 0;
#pragma unroll
      for (int w = 0; w < kCrcThreads / 32; w++) x ^= s.red[w];
      const uint32_t preset = len == block_bytes ? preset_full : gf_mul(0xFFFFFFFFu, xpow8(len));
      crc[blk] = ~(x ^ preset);
    }
    __syncthreads();
  }
}

}  // namespace

int crc_blocks_per_sm() {
  if (cudaFuncSetAttribute(k_crc32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(sizeof(CrcSmem))) != cudaSuccess)
    return 0;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_crc32, kCrcThreads, sizeof(CrcSmem)) !=
      cudaSuccess)
    return 0;
  return nb;
}

cudaError_t launch_crc32(const uint8_t *buf, uint64_t bytes, uint64_t block_bytes, uint32_t *crc,
                         int grid, cudaStream_t s) {
  k_crc32<<<grid, kCrcThreads, sizeof(CrcSmem), s>>>(buf, bytes, block_bytes, crc);
  return cudaGetLastError();
}

}  // namespace wc
