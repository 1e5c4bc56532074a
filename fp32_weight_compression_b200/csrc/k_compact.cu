// k_compact.cu -- encoder stage 3: move each chunk's payload to its final
// place in the container's exponent section (offsets from the scan), zero-padded
// to 16 bytes.  One block per chunk.
//   coded chunk: the 32 final states (front of the chunk's scratch window) and
//                the w words (back of the window, at a 2-byte aligned start;
//                realigned here with funnel shifts into 16-byte stores);
//   raw chunk:   the chunk's coded bytes (exponents; fp16 high bytes; fp8
//                exponent nibbles), re-extracted from the input
//                ("PTWM" Configuration table, compression_threshold: data that
//                does not compress is stored as it is).
#include "wc_block.cuh"
#include "wc_format.cuh"
#include "wc_planes.cuh"

namespace wc {

constexpr int kCompactThreads = 256;

// bytes [mis, mis + 16) of the 32 bytes a:b (mis even, 0..14)
__device__ __forceinline__ uint4 extract16(uint4 a, uint4 b, uint32_t mis) {
  const uint32_t sh = (mis & 3u) * 8u;
  uint32_t r0, r1, r2, r3, r4;
  switch (mis >> 2) {
    case 0: r0 = a.x; r1 = a.y; r2 = a.z; r3 = a.w; r4 = b.x; break;
    case 1: r0 = a.y; r1 = a.z; r2 = a.w; r3 = b.x; r4 = b.y; break;
    case 2: r0 = a.z; r1 = a.w; r2 = b.x; r3 = b.y; r4 = b.z; break;
    default: r0 = a.w; r1 = b.x; r2 = b.y; r3 = b.z; r4 = b.w; break;
  }
  return make_uint4(__funnelshift_r(r0, r1, sh), __funnelshift_r(r1, r2, sh),
                    __funnelshift_r(r2, r3, sh), __funnelshift_r(r3, r4, sh));
}

__device__ __forceinline__ uint32_t keep_bytes(uint32_t v, int keep) {
  if (keep >= 4) return v;
  if (keep <= 0) return 0;
  return v & ((1u << (8 * keep)) - 1u);
}

__global__ void __launch_bounds__(kCompactThreads) k_compact(const __grid_constant__ EncParams p) {
  const int tid = threadIdx.x;
  const uint32_t g = blockIdx.x;
  const EncItem &it = p.items[find_item_by_chunk(p, g)];
  const uint64_t k = g - it.chunk_base;
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);
  const uint32_t nsym = chunk_nsym(it.n, k);
  const uint64_t o0 = reinterpret_cast<const uint64_t *>(it.out + L.off_chunk_off)[k];
  const uint32_t len = reinterpret_cast<const uint32_t *>(it.out + L.off_chunk_len)[k];
  uint8_t *dst = it.out + L.off_exp + o0;

  if (len == nsym) {
    const uint32_t ngran = uint32_t(round16(nsym) / 16);
    if (is_fp8(dtype)) {
      const uint8_t *src = it.in + k * kChunk;
      for (uint32_t gi = tid; gi < ngran; gi += kCompactThreads) {
        const uint32_t v0 = gi * 16;
        uint4 e;
        if (v0 + 16 <= nsym) {
          const uint4 a = ld_nc_v4(src + v0);
          e = make_uint4(fp8_code4(a.x), fp8_code4(a.y), fp8_code4(a.z), fp8_code4(a.w));
        } else {  // ragged: exponent nibbles, zero padding bytes
          uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (uint32_t q = 0; q < 16; q++)
            if (v0 + q < nsym) w[q / 4] |= fp8_code(src[v0 + q]) << (8 * (q % 4));
          e = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *reinterpret_cast<uint4 *>(dst + v0) = e;
      }
    } else if (dtype != WC_FP32) {
      const uint16_t *src = reinterpret_cast<const uint16_t *>(it.in) + k * kChunk;
      const bool bf = dtype == WC_BF16;
      for (uint32_t gi = tid; gi < ngran; gi += kCompactThreads) {
        const uint32_t v0 = gi * 16;
        uint32_t w[8];
        if (v0 + 16 <= nsym) {
          uint4 a = ld_nc_v4(src + v0), b = ld_nc_v4(src + v0 + 8);
          w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else {
#pragma unroll
          for (int q = 0; q < 8; q++) {
            uint32_t lo = v0 + 2 * q < nsym ? src[v0 + 2 * q] : 0u;
            uint32_t hi = v0 + 2 * q + 1 < nsym ? src[v0 + 2 * q + 1] : 0u;
            w[q] = lo | (hi << 16);
          }
        }
        uint4 e;
        if (bf) {
          e.x = code4<WC_BF16>(w[0], w[1]); e.y = code4<WC_BF16>(w[2], w[3]);
          e.z = code4<WC_BF16>(w[4], w[5]); e.w = code4<WC_BF16>(w[6], w[7]);
        } else {
          e.x = code4<WC_FP16>(w[0], w[1]); e.y = code4<WC_FP16>(w[2], w[3]);
          e.z = code4<WC_FP16>(w[4], w[5]); e.w = code4<WC_FP16>(w[6], w[7]);
        }
        if (v0 + 16 > nsym) {  // zero the padding bytes
          const int keep = int(nsym - v0);
          e.x = keep_bytes(e.x, keep); e.y = keep_bytes(e.y, keep - 4);
          e.z = keep_bytes(e.z, keep - 8); e.w = keep_bytes(e.w, keep - 12);
        }
        *reinterpret_cast<uint4 *>(dst + v0) = e;
      }
    } else {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(it.in) + k * kChunk;
      for (uint32_t gi = tid; gi < ngran; gi += kCompactThreads) {
        const uint32_t v0 = gi * 16;
        uint32_t u[16];
        if (v0 + 16 <= nsym) {
#pragma unroll
          for (int q = 0; q < 4; q++) {
            uint4 a = ld_nc_v4(src + v0 + 4 * q);
            u[4 * q] = a.x; u[4 * q + 1] = a.y; u[4 * q + 2] = a.z; u[4 * q + 3] = a.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; q++) u[q] = v0 + q < nsym ? src[v0 + q] : 0u;
        }
        uint32_t e[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
          uint32_t p01 = __byte_perm(u[4 * q] << 1, u[4 * q + 1] << 1, 0x0073);
          uint32_t p23 = __byte_perm(u[4 * q + 2] << 1, u[4 * q + 3] << 1, 0x0073);
          e[q] = __byte_perm(p01, p23, 0x5410);
        }
        if (v0 + 16 > nsym) {
          const int keep = int(nsym - v0);
          e[0] = keep_bytes(e[0], keep); e[1] = keep_bytes(e[1], keep - 4);
          e[2] = keep_bytes(e[2], keep - 8); e[3] = keep_bytes(e[3], keep - 12);
        }
        *reinterpret_cast<uint4 *>(dst + v0) = make_uint4(e[0], e[1], e[2], e[3]);
      }
    }
    return;
  }

  // coded chunk
  const uint8_t *win = it.scratch + scratch_win_offset(L.nc) + k * kWin;
  if (tid < int(kStateBytes / 16))
    reinterpret_cast<uint4 *>(dst)[tid] = reinterpret_cast<const uint4 *>(win)[tid];
  const uint32_t nbytes = len - kStateBytes;  // 2w
  const uint32_t S = uint32_t(kWin) - nbytes;  // first word's byte offset in the window
  const uint32_t mis = S & 15u;
  const uint32_t A0 = S - mis;
  const uint32_t ngran = (nbytes + 15) / 16;
  for (uint32_t j = tid; j < ngran; j += kCompactThreads) {
    const uint32_t a_off = A0 + 16 * j;
    const uint4 a = __ldcg(reinterpret_cast<const uint4 *>(win + a_off));
    const uint4 b = a_off + 16 < uint32_t(kWin) ? __ldcg(reinterpret_cast<const uint4 *>(win + a_off + 16))
                                                : make_uint4(0, 0, 0, 0);
    uint4 o = extract16(a, b, mis);
    const int keep = int(nbytes) - int(16 * j);
    if (keep < 16) {
      o.x = keep_bytes(o.x, keep); o.y = keep_bytes(o.y, keep - 4);
      o.z = keep_bytes(o.z, keep - 8); o.w = keep_bytes(o.w, keep - 12);
    }
    *reinterpret_cast<uint4 *>(dst + kStateBytes + 16 * j) = o;
  }
}

cudaError_t launch_compact(const EncParams &p, cudaStream_t s) {
  if (p.total_chunks == 0) return cudaSuccess;
  k_compact<<<p.total_chunks, kCompactThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
