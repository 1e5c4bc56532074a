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
// Work split.  One CTA (16 warps) per block at a time, grid-strided over the
// blocks.  Warp w owns the w-th sixteenth of the block; inside it lane l takes
// the 16-byte pieces l, l+32, l+64, ... so that every warp load covers 512
// contiguous bytes.  A lane keeps two running registers, one over its even
// and one over its odd pieces (two independent chains of lookups in flight):
// the next piece of a chain starts 1024 bytes after the previous one began,
// so between pieces the register jumps over 1008 bytes (c -> c * x^(8*1008),
// a linear map done with four byte tables J_k) before the 16 bytes are fed
// in.  At the end each register is multiplied by x^(8 * bytes after its last
// piece) and the CTA xors the 1024 products.  For full blocks those
// multipliers are the same in every block and are computed once per launch;
// a block's ragged tail (< 16 bytes) is fed in byte by byte.
//
// Tables.  S_k[b] = raw(byte b followed by k zero bytes), k = 0..3, give one
// 4-byte step:  r ^= w;  r = S_3[r0] ^ S_2[r1] ^ S_1[r2] ^ S_0[r3]  (ri the
// bytes of r, r0 lowest); J_k[b] = (b << 8k) * x^(8*1008).  Lookups are
// data-dependent: the S tables are held 32 times over in shared memory,
// entry (k, b) of lane l at word ((k * 256 + b) * 32 + l), so every lane
// reads its own bank; the J tables (a quarter of the lookups) 16 times, lane
// l reading copy l mod 16 (at most two lanes per bank).
#include <cstdint>

#include "wc.h"
#include "wc_format.cuh"

namespace wc {
namespace {

constexpr int kCrcWarps = 16;
constexpr int kCrcThreads = 32 * kCrcWarps;
constexpr uint32_t kGenReversed = 0xEDB88320u;
constexpr uint32_t kJump = 1024 - 16;  // bytes between two pieces of one chain

struct CrcSmem {
  uint32_t srep[4 * 256 * 32];  // S tables, one copy per lane      128 KiB
  uint32_t jrep[4 * 256 * 16];  // J tables, one copy per half-warp  64 KiB
  uint32_t sbase[4 * 256];      // the tables once
  uint32_t jbase[4 * 256];
  uint32_t red[kCrcWarps];
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

__device__ __forceinline__ uint32_t byte_of(uint32_t r, int k) {
  return __byte_perm(r, 0u, 0x4440u + uint32_t(k));
}

// one 4-byte step; s = this lane's column of the S copies
__device__ __forceinline__ uint32_t step4(uint32_t r, uint32_t w, const uint32_t *s) {
  r ^= w;
  return s[(768u + byte_of(r, 0)) << 5] ^ s[(512u + byte_of(r, 1)) << 5] ^
         s[(256u + byte_of(r, 2)) << 5] ^ s[byte_of(r, 3) << 5];
}

// c * x^(8*1008); j = this lane's column of the J copies
__device__ __forceinline__ uint32_t jump(uint32_t c, const uint32_t *j) {
  return j[byte_of(c, 0) << 4] ^ j[(256u + byte_of(c, 1)) << 4] ^
         j[(512u + byte_of(c, 2)) << 4] ^ j[(768u + byte_of(c, 3)) << 4];
}

__device__ __forceinline__ uint32_t piece(uint32_t c, uint4 v, const uint32_t *s, const uint32_t *j) {
  c = jump(c, j);
  c = step4(c, v.x, s);
  c = step4(c, v.y, s);
  c = step4(c, v.z, s);
  return step4(c, v.w, s);
}

// The two registers over this lane's `cnt` pieces (even ones into ca, odd
// ones into cb); q = its first piece, the others 32 uint4 apart.
__device__ void lane_chains(const uint4 *q, uint32_t cnt, const uint32_t *s, const uint32_t *j,
                            uint32_t &ca, uint32_t &cb) {
  uint32_t a = 0, b = 0;
  const uint32_t groups = cnt >> 2;
  if (groups) {
    // four pieces in registers while the next four are on their way
    uint4 a0 = __ldg(q), a1 = __ldg(q + 32), a2 = __ldg(q + 64), a3 = __ldg(q + 96);
    for (uint32_t g = 1; g < groups; g++) {
      const uint4 *qg = q + 128 * g;
      const uint4 b0 = __ldg(qg), b1 = __ldg(qg + 32), b2 = __ldg(qg + 64), b3 = __ldg(qg + 96);
      a = piece(a, a0, s, j);
      b = piece(b, a1, s, j);
      a = piece(a, a2, s, j);
      b = piece(b, a3, s, j);
      a0 = b0;
      a1 = b1;
      a2 = b2;
      a3 = b3;
    }
    a = piece(a, a0, s, j);
    b = piece(b, a1, s, j);
    a = piece(a, a2, s, j);
    b = piece(b, a3, s, j);
  }
  for (uint32_t i = groups * 4; i < cnt; i++) {
    const uint4 v = __ldg(q + 32 * i);
    if (i & 1u) b = piece(b, v, s, j);
    else a = piece(a, v, s, j);
  }
  ca = a;
  cb = b;
}

// Bytes of the lane's share of the region after the last piece of the chain
// of parity `par` (region r0 + [0, 512 * cnt) of which the lane holds pieces
// lane + 32 i, i < cnt), counted to `len`; ~0 when that chain is empty.
__device__ __forceinline__ uint64_t after_last(uint64_t len, uint64_t r0, int lane, uint32_t cnt,
                                               uint32_t par) {
  if (cnt == 0 || (cnt == 1 && par == 1)) return ~uint64_t(0);
  const uint32_t last = ((cnt - 1) & 1u) == par ? cnt - 1 : cnt - 2;
  return len - (r0 + 16u * (uint64_t(lane) + 32u * uint64_t(last) + 1u));
}

__global__ void __launch_bounds__(kCrcThreads, 1)
k_crc32(const uint8_t *__restrict__ buf, uint64_t bytes, uint64_t block_bytes,
        uint32_t *__restrict__ crc) {
  CrcSmem &sm = *reinterpret_cast<CrcSmem *>(crc_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid < 256) {
    uint32_t r = uint32_t(tid);
    for (int i = 0; i < 8; i++) r = (r >> 1) ^ (kGenReversed & (0u - (r & 1u)));
    sm.sbase[tid] = r;
  }
  {
    const uint32_t x496 = xpow8(kJump);
    for (int i = tid; i < 1024; i += kCrcThreads)
      sm.jbase[i] = gf_mul(uint32_t(i & 255) << (8 * (i >> 8)), x496);
  }
  __syncthreads();
  if (tid < 256) {
    uint32_t r = sm.sbase[tid];
    for (int k = 1; k < 4; k++) {
      r = sm.sbase[r & 0xFFu] ^ (r >> 8);  // one more zero byte
      sm.sbase[k * 256 + tid] = r;
    }
  }
  __syncthreads();
  for (int i = tid; i < 4 * 256 * 32; i += kCrcThreads) sm.srep[i] = sm.sbase[i >> 5];
  for (int i = tid; i < 4 * 256 * 16; i += kCrcThreads) sm.jrep[i] = sm.jbase[i >> 4];
  __syncthreads();

  const uint32_t *s = sm.srep + lane;
  const uint32_t *j = sm.jrep + (lane & 15);
  const uint64_t nblocks = (bytes + block_bytes - 1) / block_bytes;
  const uint64_t region = block_bytes / kCrcWarps;  // a multiple of 512
  const uint32_t cnt_full = uint32_t(region / 512);
  // full blocks: bytes after each chain's last piece, and the preset's image
  const uint64_t r0 = uint64_t(warp) * region;
  const uint64_t da = after_last(block_bytes, r0, lane, cnt_full, 0);
  const uint64_t db = after_last(block_bytes, r0, lane, cnt_full, 1);
  const uint32_t mul_a = xpow8(da);
  const uint32_t mul_b = db == ~uint64_t(0) ? 0u : xpow8(db);
  const uint32_t preset_full = gf_mul(0xFFFFFFFFu, xpow8(block_bytes));

  for (uint64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const uint64_t start = blk * block_bytes;
    const uint64_t len = bytes - start < block_bytes ? bytes - start : block_bytes;
    const uint8_t *rb = buf + start + r0;
    uint32_t part = 0;
    if (len == block_bytes) {
      uint32_t ca, cb;
      lane_chains(reinterpret_cast<const uint4 *>(rb) + lane, cnt_full, s, j, ca, cb);
      if (ca) part = gf_mul(ca, mul_a);
      if (cb) part ^= gf_mul(cb, mul_b);
    } else if (len > r0) {
      // the ragged block: this warp's share may be short or end in a tail
      const uint64_t rlen = len - r0 < region ? len - r0 : region;
      const uint32_t np = uint32_t(rlen >> 4);
      const uint32_t cnt = np > uint32_t(lane) ? (np - uint32_t(lane) + 31) / 32 : 0;
      if (cnt) {
        uint32_t ca, cb;
        lane_chains(reinterpret_cast<const uint4 *>(rb) + lane, cnt, s, j, ca, cb);
        if (ca) part = gf_mul(ca, xpow8(after_last(len, r0, lane, cnt, 0)));
        if (cb) part ^= gf_mul(cb, xpow8(after_last(len, r0, lane, cnt, 1)));
      }
      const uint32_t tail = uint32_t(rlen & 15u);
      if (tail && lane == 0) {
        uint32_t c = 0;
        for (uint32_t i = 0; i < tail; i++)
          c = s[((c ^ __ldg(rb + 16u * np + i)) & 0xFFu) << 5] ^ (c >> 8);
        part ^= gf_mul(c, xpow8(len - (r0 + rlen)));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) part ^= __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (lane == 0) sm.red[warp] = part;
    __syncthreads();
    if (tid == 0) {
      uint32_t x = 0;
#pragma unroll
      for (int w = 0; w < kCrcWarps; w++) x ^= sm.red[w];
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
