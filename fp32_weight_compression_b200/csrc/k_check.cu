// k_check.cu -- exhaustive check, on the GPU, of the encoder's division by
// the symbol frequency (wc_coder.cuh): the coding step must equal
// (x / f) 4096 + x % f + cum for every frequency f and every renormalised
// state x < f 2^20, computed with the very function the encoder runs.
//
// The states checked are those the encoder can divide: every state is >= 2^16
// before a step, and a state at or above f 2^20 loses 16 bits first, so the
// divided state x lies in [16 f, f 2^20).  Block (bx, fy) takes frequency
// f_first + fy and the states x = 16 f + bx * 256 + tid, + gridDim.x * 256,
// ...; the true quotient and remainder are carried
// along the stride (one division per thread, at the start), so each state
// costs a coding step, a comparison and a few adds.
#include <cstdint>

#include "wc.h"
#include "wc_coder.cuh"
#include "wc_diag.h"
#include "wc_format.cuh"

namespace wc {

constexpr int kCheckThreads = 256;
constexpr int kCheckBlocksPerF = 64;

template <bool W>
__global__ void __launch_bounds__(kCheckThreads) k_check_division(uint32_t f_first,
                                                                  unsigned long long *res) {
  const uint32_t f = f_first + blockIdx.y;
  const uint32_t cum = 0;
  uint4 e;
  uint32_t bias;
  coder_entry(f, cum, W, e, bias);
  const uint32_t limit = (f << 20) - 1;  // the largest state coded with f (xmax)
  const uint32_t stride = gridDim.x * kCheckThreads;
  uint32_t x = 16 * f + blockIdx.x * kCheckThreads + threadIdx.x;
  if (x > limit) return;
  uint32_t q = x / f, r = x % f;
  const uint32_t qs = stride / f, rs = stride % f;
  unsigned long long bad = 0;
  for (;;) {
    const uint32_t got = advance<W>(x, e, W ? bias : 0u);
    const uint32_t want = q * kProbScale + r + cum;
    if (got != want) {
      if (bad == 0) atomicCAS(res + 1, 0ull, (static_cast<unsigned long long>(f) << 32) | x);
      bad++;
    }
    if (limit - x < stride) break;
    x += stride;
    q += qs;
    r += rs;
    if (r >= f) {
      r -= f;
      q++;
    }
  }
  if (bad) atomicAdd(res, bad);
}

}  // namespace wc

extern "C" int32_t wc_check_coder_division(int32_t wide, uint32_t f_first, uint32_t f_last,
                                           uint64_t *d_result, void *stream) {
  if (d_result == nullptr || (reinterpret_cast<uintptr_t>(d_result) & 7u) != 0) return WC_ERR_INVALID_ARG;
  if (f_first < 1 || f_last < f_first || f_last > 4095 || (!wide && f_last > 2048))
    return WC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(d_result, 0, 2 * sizeof(uint64_t), s) != cudaSuccess) return WC_ERR_CUDA;
  const dim3 grid(wc::kCheckBlocksPerF, f_last - f_first + 1);
  auto *res = reinterpret_cast<unsigned long long *>(d_result);
  if (wide) wc::k_check_division<true><<<grid, wc::kCheckThreads, 0, s>>>(f_first, res);
  else wc::k_check_division<false><<<grid, wc::kCheckThreads, 0, s>>>(f_first, res);
  return cudaGetLastError() == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}
