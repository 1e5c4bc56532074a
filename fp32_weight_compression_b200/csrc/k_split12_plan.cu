// k_split12_plan.cu -- the serving plan of a Split12 container (wc12_plan):
// its exceptions grouped by the tiles of wc12_linear (128 weight rows x 64
// values of K), layout in wc12_plan.cuh.  Built once per weight matrix, four
// launches on one stream:
//   k12p_init   checks the container's header against N, K and ne, writes
//               the plan's header and zeroes the bucket counts;
//   k12p_count  one block per chunk: counts each exception into its bucket;
//   k12p_scan   one block: the counts become the buckets' starts;
//   k12p_fill   one block per chunk: places each exception in its bucket
//               (a cursor per bucket), after which start[i] has moved on to
//               the next bucket's start, start[i + 1] in the plan's terms
//               since the counts are kept one place up.
// A container that fails a check leaves a plan whose magic is 0 (refused by
// wc12_linear_planned) and WC_ERR_CORRUPT in *status.
#include <cstdint>

#include "wc.h"
#include "wc12_plan.cuh"
#include "wc_split12.cuh"
#include "wc_split12.h"

namespace wc12p {

using wc12::kChunk;

struct PlanParams {
  const uint8_t *w;
  uint64_t w_bytes;
  uint8_t *plan;
  uint32_t N, K;
  uint64_t ne;
  int32_t *status;
};

__device__ __forceinline__ void report(int32_t *status, int32_t code) { atomicCAS(status, 0, code); }

// a corrupt container: the plan is marked invalid and the status set
__device__ __forceinline__ void corrupt(const PlanParams &p) {
  reinterpret_cast<volatile uint32_t *>(p.plan)[0] = 0u;
  report(p.status, WC_ERR_CORRUPT);
}

// The container header, checked against an N x K matrix with ne exceptions.
__device__ bool container_ok(const PlanParams &p, wc12::Lay &L) {
  const uint32_t *h32 = reinterpret_cast<const uint32_t *>(p.w);
  const uint64_t *h64 = reinterpret_cast<const uint64_t *>(p.w);
  const uint64_t n = uint64_t(p.N) * p.K;
  const uint32_t kk = h32[1] >> 24;
  if (h32[0] != wc12::kMagic || (h32[1] & 0xFFFFFFu) != (1u | (1u << 16)) || kk < 1 || kk > 16 ||
      h64[1] != n || h64[3] != p.ne || h32[4] != uint32_t(kChunk))
    return false;
  L = wc12::lay(n, p.ne);
  return h32[5] == uint32_t(L.nc) && h64[4] == L.off_idx && h64[5] == L.off_lo && h64[6] == L.off_exc &&
         h64[7] == L.total && L.total <= p.w_bytes;
}

__device__ __forceinline__ bool plan_valid(const PlanParams &p) {
  return reinterpret_cast<const volatile uint32_t *>(p.plan)[0] == kMagic;
}

__global__ void k12p_init(const __grid_constant__ PlanParams p) {
  const PlanLay P = plan_lay(p.N, p.K, p.ne);
  uint32_t *start = reinterpret_cast<uint32_t *>(p.plan + kStartOff);
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i <= P.buckets;
       i += uint64_t(gridDim.x) * blockDim.x)
    start[i] = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    wc12::Lay L;
    const bool ok = container_ok(p, L);
    uint32_t *h32 = reinterpret_cast<uint32_t *>(p.plan);
    uint64_t *h64 = reinterpret_cast<uint64_t *>(p.plan);
    h32[0] = ok ? kMagic : 0u;
    h32[1] = 1;
    h32[2] = p.N;
    h32[3] = p.K;
    h64[2] = p.ne;
    h64[3] = P.buckets;
    if (!ok) report(p.status, WC_ERR_CORRUPT);
  }
}

// The exceptions of chunk blockIdx.x, each with its bucket; FILL: placed,
// else counted (into start[bucket + 1]).
template <bool FILL>
__global__ void __launch_bounds__(256) k12p_chunk(const __grid_constant__ PlanParams p) {
  if (!plan_valid(p)) return;
  const uint64_t n = uint64_t(p.N) * p.K;
  const wc12::Lay L = wc12::lay(n, p.ne);
  const uint64_t c = blockIdx.x;
  const uint64_t *exc_off = reinterpret_cast<const uint64_t *>(p.w + wc12::kExcOffOff);
  const uint16_t *exc_pos = reinterpret_cast<const uint16_t *>(p.w + L.off_exc);
  const uint8_t *exc_val = p.w + L.off_excval;
  const PlanLay P = plan_lay(p.N, p.K, p.ne);
  uint32_t *start = reinterpret_cast<uint32_t *>(p.plan + kStartOff);
  uint32_t *ent = reinterpret_cast<uint32_t *>(p.plan + P.off_ent);
  const uint64_t e0 = exc_off[c], e1 = exc_off[c + 1];
  if (e0 > e1 || e1 > p.ne || (c == 0 && e0 != 0) || (c + 1 == L.nc && e1 != p.ne)) {
    if (threadIdx.x == 0) corrupt(p);
    return;
  }
  const uint64_t cnt = n - c * kChunk < kChunk ? n - c * kChunk : kChunk;
  const uint32_t S = p.K / kValues;
  for (uint64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const uint32_t pos = exc_pos[e];
    if (pos >= cnt) {
      corrupt(p);
      continue;
    }
    const uint64_t f = c * kChunk + pos;
    const uint64_t row = f / p.K, col = f % p.K;
    const uint64_t bucket = (row / kRows) * S + col / kValues;
    if (!FILL) {
      atomicAdd(&start[bucket + 1], 1u);
    } else {
      const uint32_t slot = atomicAdd(&start[bucket + 1], 1u);
      if (slot < p.ne)
        ent[slot] = pack_entry(uint32_t(col % kValues), uint32_t(row % kRows), exc_val[e]);
      else
        corrupt(p);
    }
  }
}

// start[1 .. buckets]: counts -> exclusive prefix (start[1] = 0), one block
__global__ void __launch_bounds__(1024) k12p_scan(const __grid_constant__ PlanParams p) {
  if (!plan_valid(p)) return;
  __shared__ uint32_t warp_sum[32];
  __shared__ uint32_t carry_s;
  const PlanLay P = plan_lay(p.N, p.K, p.ne);
  uint32_t *cnt = reinterpret_cast<uint32_t *>(p.plan + kStartOff) + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (uint64_t base = 0; base < P.buckets; base += 1024) {
    const uint64_t i = base + tid;
    const uint32_t v = i < P.buckets ? cnt[i] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t ws = warp_sum[lane];
      uint32_t wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      warp_sum[lane] = wi - ws;  // exclusive prefix of the warps
    }
    __syncthreads();
    const uint32_t carry = carry_s;
    if (i < P.buckets) cnt[i] = carry + warp_sum[warp] + incl - v;
    __syncthreads();
    if (tid == 1023) carry_s = carry + warp_sum[warp] + incl;
    __syncthreads();
  }
}

}  // namespace wc12p

extern "C" {

uint64_t wc12_plan_bytes(uint32_t N, uint32_t K, uint64_t ne) {
  return wc12p::plan_lay(N, K, ne).total;
}

int32_t wc12_plan(const void *d_w, uint64_t w_bytes, uint32_t N, uint32_t K, uint64_t ne, void *d_plan,
                  uint64_t plan_bytes, int32_t *d_status, void *stream) {
  auto aligned = [](const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; };
  if (d_w == nullptr || d_plan == nullptr || d_status == nullptr) return WC_ERR_INVALID_ARG;
  if (!aligned(d_w, 16) || !aligned(d_plan, 16) || !aligned(d_status, 4)) return WC_ERR_INVALID_ARG;
  if (N == 0 || K == 0 || N % wc12p::kRows != 0 || K % wc12p::kValues != 0) return WC_ERR_INVALID_ARG;
  const uint64_t n = uint64_t(N) * K;
  if (n > wc12::kMaxN || ne > n || ne >= (uint64_t(1) << 32)) return WC_ERR_INVALID_ARG;
  const wc12::Lay L = wc12::lay(n, ne);
  if (w_bytes < L.total) return WC_ERR_INVALID_ARG;  // too short for its header's layout
  if (plan_bytes < wc12p::plan_lay(N, K, ne).total) return WC_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  wc12p::PlanParams p{static_cast<const uint8_t *>(d_w), w_bytes, static_cast<uint8_t *>(d_plan), N, K, ne,
                      d_status};
  const unsigned chunks = unsigned(L.nc);
  wc12p::k12p_init<<<256, 256, 0, s>>>(p);
  if (chunks > 0) wc12p::k12p_chunk<false><<<chunks, 256, 0, s>>>(p);
  wc12p::k12p_scan<<<1, 1024, 0, s>>>(p);
  if (chunks > 0) wc12p::k12p_chunk<true><<<chunks, 256, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

}  // extern "C"
