// k_hist.cu -- encoder stage 1: container header, per-tensor histogram of
// the coded bytes, and the 12-bit frequency table.
//
//  k_prep   one block per tensor: clears the tensor's scratch counters and
//           writes the fixed header fields and the zero padding of the
//           container (everything that depends on n alone).
//  k_hist   one block (512 threads) per tile of up to 4 chunks: counts the
//           tile's coded bytes into a shared [symbol][lane] histogram
//           (wc_hist.cuh), adds them to the tensor's histogram, and the last
//           tile of a tensor turns the counts into the table (the table
//           rule and its closed-form evaluation are described in
//           wc_hist.cuh).  The whole GPU reads the input at memory speed.
#include "wc_block.cuh"
#include "wc_format.cuh"
#include "wc_hist.cuh"
#include "wc_planes.cuh"

namespace wc {

// ---------------------------------------------------------------------------
// Header fields, padding and scratch counters (one block per tensor).
__global__ void __launch_bounds__(256) k_prep(const __grid_constant__ EncParams p) {
  const EncItem &it = p.items[blockIdx.x];
  const int tid = threadIdx.x;
  const int dtype = int(it.dtype);
  const Layout L = make_layout(it.n, dtype);
  uint8_t *out = it.out;

  uint64_t *hist = reinterpret_cast<uint64_t *>(it.scratch + kScrHist);
  uint32_t *ctr = reinterpret_cast<uint32_t *>(it.scratch + kScrCtr);
  hist[tid] = 0;
  if (tid < 4) ctr[tid] = 0;

  // table: all zero until the last histogram tile writes it (n = 0 keeps it)
  reinterpret_cast<uint16_t *>(out + kFreqOffset)[tid] = 0;

  if (tid == 0) {
    uint32_t *h32 = reinterpret_cast<uint32_t *>(out);
    uint64_t *h64 = reinterpret_cast<uint64_t *>(out);
    h32[0] = 0x315A4357u;  // "WCZ1"
    h32[1] = kVersion | (uint32_t(dtype) << 16) | (kLanes << 24);
    h64[1] = it.n;
    h32[4] = kChunk;
    h32[5] = uint32_t(L.nc);
    h32[6] = kProbBits;  // u16 12, u16 0
    h32[7] = 0;
    h64[4] = L.off_raw;
    h64[5] = L.off_exp;
    if (it.n == 0) {
      h64[6] = 0;
      h64[7] = L.off_exp;
      *reinterpret_cast<uint64_t *>(out + L.off_chunk_off) = 0;
      *it.out_size = L.off_exp;
    }
  }
  // zero padding: after the chunk-length table, and after each raw plane
  if (tid < 16) {
    uint64_t a = L.off_chunk_len + 4 * L.nc + tid;
    if (a < L.off_raw) out[a] = 0;
    if (dtype != WC_FP32) {
      const uint64_t raw_bytes = is_fp8(dtype) ? (it.n + 1) / 2 : it.n;
      uint64_t b = L.off_raw + raw_bytes + tid;
      if (b < L.off_exp) out[b] = 0;
    } else {
      uint64_t b = L.off_raw + (it.n + 7) / 8 + tid;
      if (b < L.off_mant) out[b] = 0;
      uint64_t c = L.off_mant + 3 * it.n + tid;
      if (c < L.off_exp) out[c] = 0;
    }
  }
}

// ---------------------------------------------------------------------------
constexpr int kHistThreads = 512;

__global__ void __launch_bounds__(kHistThreads, 2) k_hist(const __grid_constant__ EncParams p) {
  __shared__ __align__(16) uint32_t sh[256 * 32];  // [symbol][lane]
  __shared__ uint64_t red[kHistThreads / 32 + 1];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const uint32_t b = blockIdx.x;
  const EncItem &it = p.items[find_item_by_hist(p, b)];
  const uint64_t tile = b - it.hist_base;
  for (int i = tid; i < 256 * 32 / 4; i += kHistThreads)
    reinterpret_cast<uint4 *>(sh)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  count_tile<kHistThreads>(it, tile, sh);
  __syncthreads();
  uint64_t *ghist = reinterpret_cast<uint64_t *>(it.scratch + kScrHist);
  if (tid < 256) {
    uint32_t sum = 0;
#pragma unroll 8
    for (int j = 0; j < 32; j++) sum += sh[(tid << 5) | ((j + tid) & 31)];
    if (sum) atomicAdd(reinterpret_cast<unsigned long long *>(&ghist[tid]),
                       static_cast<unsigned long long>(sum));
    __threadfence();
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t *ctr = reinterpret_cast<uint32_t *>(it.scratch + kScrCtr);
    const uint64_t nc = num_chunks(it.n);
    const uint32_t nt = uint32_t((nc + kHistChunks - 1) / kHistChunks);
    s_last = (atomicAdd(&ctr[0], 1u) == nt - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  publish_table<kHistThreads>(it, red);
}

cudaError_t launch_prep(const EncParams &p, cudaStream_t s) {
  k_prep<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hist(const EncParams &p, cudaStream_t s) {
  if (p.total_hist_blocks == 0) return cudaSuccess;
  k_hist<<<p.total_hist_blocks, kHistThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
