// k_encode.cu -- encoder stage 2: plane split + rANS coding per chunk, and the
// exclusive scan of chunk sizes into the container's offset table.
//
// One warp codes one 65,536-value chunk (one rANS state per lane, symbol i in
// lane i mod 32).  The warp walks its chunk backwards in groups of 512 values
// (16 steps): each lane loads its 16 consecutive values, writes their raw
// planes straight into the container's raw section (bf16: the sign+mantissa
// byte; fp32: sign bits and 3 little-endian mantissa bytes -- "PTWM" How it
// works 1-2, "SMEF" pass3_streams.py), and parks their exponent bytes in shared
// memory, where step t reads byte 32 t + lane.  Coding a symbol s with
// frequency f from state x (12-bit table, L = 2^16, 16-bit words):
//   if x >= f 2^20: emit x & 0xFFFF, x >>= 16;   x = (x / f) 4096 + x % f + cum_s
// with x / f computed exactly as floor(x m / 2^64), m = ceil(2^64 / f) split in
// two 32-bit halves (two integer multiply-adds; see publish_table).  The lanes
// that emit at a step form one block of the word stream, in ascending lane
// order, placed with __ballot_sync / __popc prefix offsets; blocks are laid
// down back to front, so the decoder (which runs the steps forwards) reads
// them in order.  A chunk stops coding as soon as 128 + 2w >= nsym: it will be
// stored raw ("PTWM" Configuration table, compression_threshold).
//
// The last warp to finish a tensor scans the tensor's chunk lengths into
// chunk_off[] (16-byte rounded) and chunk_len[] and completes the header.
#include "wc_block.cuh"
#include "wc_format.cuh"

namespace wc {

constexpr int kCoderThreads = kCoderWarps * 32;

// 16 values of one lane, as raw 32-bit words (bf16: 8 words, fp32: 16 words).
template <int DT>
struct Vals {
  uint32_t w[DT == WC_BF16 ? 8 : 16];
};

template <int DT>
__device__ __forceinline__ void load_vals(const uint8_t *src, uint32_t nv, Vals<DT> &v) {
  if (nv == 16) {
#pragma unroll
    for (int q = 0; q < (DT == WC_BF16 ? 2 : 4); q++) {
      uint4 a = ld_nc_v4(src + 16 * q);
      v.w[4 * q + 0] = a.x; v.w[4 * q + 1] = a.y; v.w[4 * q + 2] = a.z; v.w[4 * q + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < (DT == WC_BF16 ? 8 : 16); q++) v.w[q] = 0;
    if (DT == WC_BF16) {
      const uint16_t *s16 = reinterpret_cast<const uint16_t *>(src);
      for (uint32_t j = 0; j < nv; j++) {
        uint32_t b = s16[j];
        // place value j in half (j & 1) of word j >> 1 (dynamic index kept in
        // a small loop to stay in registers)
#pragma unroll
        for (int q = 0; q < 8; q++)
          if (q == int(j >> 1)) v.w[q] |= b << (16 * (j & 1));
      }
    } else {
      const uint32_t *s32 = reinterpret_cast<const uint32_t *>(src);
#pragma unroll
      for (int q = 0; q < 16; q++)
        if (uint32_t(q) < nv) v.w[q] = s32[q];
    }
  }
}

// Exponent bytes of the 16 values, packed little-endian into a uint4.
template <int DT>
__device__ __forceinline__ uint4 exponents(const Vals<DT> &v) {
  uint32_t e[4];
  if (DT == WC_BF16) {
    // bf16 word = [v1 : v0]; exponent of a value = bits 7..14 of its half
#pragma unroll
    for (int q = 0; q < 4; q++)
      e[q] = __byte_perm(v.w[2 * q] >> 7, v.w[2 * q + 1] >> 7, 0x6420);
  } else {
    // fp32: exponent = byte 3 of (u << 1)
#pragma unroll
    for (int q = 0; q < 4; q++) {
      uint32_t p01 = __byte_perm(v.w[4 * q] << 1, v.w[4 * q + 1] << 1, 0x0073);
      uint32_t p23 = __byte_perm(v.w[4 * q + 2] << 1, v.w[4 * q + 3] << 1, 0x0073);
      e[q] = __byte_perm(p01, p23, 0x5410);
    }
  }
  return make_uint4(e[0], e[1], e[2], e[3]);
}

// Raw planes of the 16 values (value index vg within the tensor) into the
// container's raw section.
template <int DT>
__device__ __forceinline__ void store_raw(uint8_t *out, const Layout &L, uint64_t vg, uint32_t nv,
                                          const Vals<DT> &v) {
  if (DT == WC_BF16) {
    // sm byte = sign << 7 | mantissa = (high byte & 0x80) | (low byte & 0x7F)
    uint32_t sm[4];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      uint32_t lo = __byte_perm(v.w[2 * q], v.w[2 * q + 1], 0x6420);
      uint32_t hi = __byte_perm(v.w[2 * q], v.w[2 * q + 1], 0x7531);
      sm[q] = (lo & 0x7F7F7F7Fu) | (hi & 0x80808080u);
    }
    uint8_t *dst = out + L.off_raw + vg;
    if (nv == 16) {
      st_cs_v4(dst, make_uint4(sm[0], sm[1], sm[2], sm[3]));
    } else {
      for (uint32_t j = 0; j < nv; j++) {
        uint32_t word = 0;
#pragma unroll
        for (int q = 0; q < 4; q++)
          if (q == int(j >> 2)) word = sm[q];
        dst[j] = uint8_t(word >> (8 * (j & 3)));
      }
    }
  } else {
    uint32_t sbits = 0;
#pragma unroll
    for (int j = 0; j < 16; j++) sbits |= (v.w[j] >> 31) << j;
    uint32_t mw[12];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      uint32_t m0 = v.w[4 * q] & 0x7FFFFFu, m1 = v.w[4 * q + 1] & 0x7FFFFFu;
      uint32_t m2 = v.w[4 * q + 2] & 0x7FFFFFu, m3 = v.w[4 * q + 3] & 0x7FFFFFu;
      mw[3 * q + 0] = m0 | (m1 << 24);
      mw[3 * q + 1] = (m1 >> 8) | (m2 << 16);
      mw[3 * q + 2] = (m2 >> 16) | (m3 << 8);
    }
    uint8_t *sdst = out + L.off_raw + vg / 8;
    uint8_t *mdst = out + L.off_mant + 3 * vg;
    if (nv == 16) {
      *reinterpret_cast<uint16_t *>(sdst) = uint16_t(sbits);
      st_cs_v4(mdst, make_uint4(mw[0], mw[1], mw[2], mw[3]));
      st_cs_v4(mdst + 16, make_uint4(mw[4], mw[5], mw[6], mw[7]));
      st_cs_v4(mdst + 32, make_uint4(mw[8], mw[9], mw[10], mw[11]));
    } else {
      // padding values are zero, so their sign bits are zero
      sdst[0] = uint8_t(sbits);
      if (nv > 8) sdst[1] = uint8_t(sbits >> 8);
      for (uint32_t j = 0; j < 3 * nv; j++) {
        uint32_t word = 0;
#pragma unroll
        for (int q = 0; q < 12; q++)
          if (q == int(j >> 2)) word = mw[q];
        mdst[j] = uint8_t(word >> (8 * (j & 3)));
      }
    }
  }
}

// One coding step of one lane.  CHECK: the step may hold lanes past nsym.
template <bool CHECK>
__device__ __forceinline__ void code_step(uint32_t &x, uint32_t &tail, uint16_t *win16,
                                          const uint4 *tab, const uint32_t *bias, uint32_t s,
                                          bool valid, uint32_t lt) {
  const uint4 te = tab[s];
  const uint32_t bi = bias[s];
  const bool emit = (CHECK ? valid : true) && x > te.z;
  const uint32_t m = __ballot_sync(0xffffffffu, emit);
  const uint32_t k = __popc(m);
  if (emit) {
    win16[tail - k + __popc(m & lt)] = uint16_t(x);
    x >>= 16;
  }
  tail -= k;
  if (!CHECK || valid) {
    const uint32_t qlo = __umulhi(x, te.x);
    const uint64_t prod = uint64_t(x) * te.y + qlo;
    const uint32_t q = uint32_t(prod >> 32);
    x = x + q * te.w + bi;
  }
}

template <int DT>
__device__ __forceinline__ void code_chunk(const EncItem &it, const Layout &L, uint64_t k,
                                           const uint4 *tab, const uint32_t *bias, uint8_t *ebuf) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const uint64_t nc = L.nc;
  const uint32_t nsym = chunk_nsym(it.n, k);
  const int ngroups = int((nsym + kGroupValues - 1) / kGroupValues);
  constexpr uint32_t elem = DT == WC_BF16 ? 2 : 4;
  const uint8_t *src = it.in + (k * kChunk) * elem;
  uint8_t *win = it.scratch + scratch_win_offset(nc) + k * kWin;
  uint16_t *win16 = reinterpret_cast<uint16_t *>(win);

  uint32_t x = kStateLow;
  uint32_t tail = kWinWords;
  bool bail = false;

  auto lane_nv = [&](int G) -> uint32_t {
    int64_t r = int64_t(nsym) - (int64_t(G) * kGroupValues + 16 * lane);
    return r <= 0 ? 0u : (r >= 16 ? 16u : uint32_t(r));
  };

  Vals<DT> cur, nxt;
  {
    const int G = ngroups - 1;
    const uint32_t nv = lane_nv(G);
    if (nv) load_vals<DT>(src + (uint64_t(G) * kGroupValues + 16 * lane) * elem, nv, cur);
    else {
#pragma unroll
      for (int q = 0; q < (DT == WC_BF16 ? 8 : 16); q++) cur.w[q] = 0;
    }
  }
  for (int G = ngroups - 1; G >= 0; --G) {
    const uint32_t nv = lane_nv(G);
    const uint64_t vg = k * kChunk + uint64_t(G) * kGroupValues + 16 * lane;
    if (nv) store_raw<DT>(it.out, L, vg, nv, cur);
    uint4 e = exponents<DT>(cur);
    *reinterpret_cast<uint4 *>(ebuf + 16 * lane) = e;
    if (G > 0) load_vals<DT>(src + (uint64_t(G - 1) * kGroupValues + 16 * lane) * elem, 16, nxt);
    __syncwarp();
    if (!bail) {
      const uint32_t gbase = uint32_t(G) * kGroupValues;
      if (gbase + kGroupValues <= nsym) {
#pragma unroll
        for (int t = kStepsPerGroup - 1; t >= 0; --t)
          code_step<false>(x, tail, win16, tab, bias, ebuf[32 * t + lane], true, lt);
      } else {
        const int steps = int((nsym - gbase + 31) / 32);
        for (int t = steps - 1; t >= 0; --t) {
          const bool valid = gbase + 32 * t + lane < nsym;
          code_step<true>(x, tail, win16, tab, bias, ebuf[32 * t + lane], valid, lt);
        }
      }
      if (kStateBytes + 2 * (kWinWords - tail) >= nsym) bail = true;
    }
    __syncwarp();
    if (G > 0) cur = nxt;
  }

  const uint32_t w = kWinWords - tail;
  const bool raw = bail || (kStateBytes + 2 * w >= nsym);
  const uint32_t len = raw ? nsym : kStateBytes + 2 * w;
  if (!raw) reinterpret_cast<uint32_t *>(win)[lane] = x;
  uint32_t *lens = reinterpret_cast<uint32_t *>(it.scratch + kScrLen);
  if (lane == 0) lens[k] = len;
}

__global__ void __launch_bounds__(kCoderThreads, 4) k_coder(const __grid_constant__ EncParams p) {
  __shared__ uint4 s_tab[256];
  __shared__ uint32_t s_bias[256];
  __shared__ __align__(16) uint8_t s_ebuf[kCoderWarps][kGroupValues];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t b = blockIdx.x;
  const EncItem &it = p.items[find_item_by_block(p, b)];
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);

  s_tab[tid] = reinterpret_cast<const uint4 *>(it.scratch + kScrTab)[tid];
  s_bias[tid] = reinterpret_cast<const uint32_t *>(it.scratch + kScrBias)[tid];
  __syncthreads();

  const uint64_t k = uint64_t(b - it.block_base) * kCoderWarps + warp;
  if (k >= L.nc) return;
  if (dtype == WC_BF16) code_chunk<WC_BF16>(it, L, k, s_tab, s_bias, s_ebuf[warp]);
  else code_chunk<WC_FP32>(it, L, k, s_tab, s_bias, s_ebuf[warp]);

  // last warp of the tensor: offset table and the rest of the header
  __threadfence();
  uint32_t prev = 0;
  if (lane == 0) prev = atomicAdd(reinterpret_cast<uint32_t *>(it.scratch + kScrCtr) + 1, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != uint32_t(L.nc - 1)) return;
  __threadfence();
  const uint32_t *lens = reinterpret_cast<const uint32_t *>(it.scratch + kScrLen);
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
