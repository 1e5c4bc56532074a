// wc_block.cuh -- warp/block reductions, scans and small PTX wrappers used by
// the codec kernels.
#pragma once

#include <cstdint>

namespace wc {

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    uint64_t u = __shfl_xor_sync(0xffffffffu, v, o);
    v = u > v ? u : v;
  }
  return v;
}

// Inclusive scan over a warp.
__device__ __forceinline__ uint32_t warp_incl_scan_u32(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Block-wide reductions.  Every thread of the block must call them; `sm`
// points at (NT/32 + 1) u64 of shared memory that is free between calls.
template <int NT>
__device__ __forceinline__ uint64_t block_sum_u64(uint64_t v, uint64_t *sm) {
  constexpr int W = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_u64(v);
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint64_t t = lane < W ? sm[lane] : 0;
    t = warp_sum_u64(t);
    if (lane == 0) sm[W] = t;
  }
  __syncthreads();
  uint64_t r = sm[W];
  __syncthreads();
  return r;
}

template <int NT>
__device__ __forceinline__ uint64_t block_max_u64(uint64_t v, uint64_t *sm) {
  constexpr int W = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max_u64(v);
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint64_t t = lane < W ? sm[lane] : 0;
    t = warp_max_u64(t);
    if (lane == 0) sm[W] = t;
  }
  __syncthreads();
  uint64_t r = sm[W];
  __syncthreads();
  return r;
}

// Exclusive scan over the block (thread order).  `sm`: NT/32 + 1 u64.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan_u64(uint64_t v, uint64_t *sm) {
  constexpr int W = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t incl = warp_incl_scan_u64(v);
  if (lane == 31) sm[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint64_t t = lane < W ? sm[lane] : 0;
    uint64_t ti = warp_incl_scan_u64(t);
    if (lane < W) sm[lane] = ti - t;  // exclusive prefix of warp totals
  }
  __syncthreads();
  uint64_t r = sm[warp] + incl - v;
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// cp.async (global -> shared, 16 bytes, bypassing L1).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, uint32_t src_bytes) {
  uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async16_s(uint32_t smem_dst, const void *gmem_src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_dst), "l"(gmem_src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Streaming loads / stores.
__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_cs_v2(void *p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};\n" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_cs_v4(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// A release store at GPU scope (a flag another block may poll).
__device__ __forceinline__ void st_release_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

}  // namespace wc
