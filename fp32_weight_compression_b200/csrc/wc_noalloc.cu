// wc_noalloc.cu -- wc_encode_noalloc: encoding for callers that cannot
// allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) at
// the point where they want to compress a tensor: a runtime that owns all
// device memory through a fixed, pre-planned arena and forbids allocations
// outside it; a plug-in that another framework calls with only its input and
// output buffers; a latency-critical path that cannot afford cudaMalloc's
// implicit device-wide synchronisation.  wc_encode needs a scratch buffer the
// caller provides; this entry point instead uses a scratch area that the
// library itself holds in device memory, so the caller passes only the input
// and the output.
//
// The scratch area is one file-scope __device__ array of
// WC_NOALLOC_SCRATCH_BYTES.  Every GPU that loads this library holds one copy
// of it from the moment the library's module is loaded on that GPU until the
// process exits.  All calls on a GPU share that one copy.
#include <mutex>

#include "wc.h"
#include "wc_format.cuh"

namespace {

// The library-held scratch (see the header comment of wc_encode_noalloc).
static __device__ __align__(256) uint8_t g_noalloc_scratch[WC_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on each device, looked up once per
// device with that device current (in host code the symbol's name is only a
// host-side stand-in, never a device address).
void *scratch_address(int32_t *err) {
  static std::mutex mu;
  static void *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *err = WC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *err = WC_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *err = WC_OK;
  return addr[dev];
}

}  // namespace

extern "C" WC_API int32_t wc_encode_noalloc(const void *d_in, uint64_t n, int32_t dtype, void *d_out,
                                            uint64_t out_cap, uint64_t *d_out_size, void *stream) {
  const uint64_t need = wc_scratch_bytes(n, dtype);
  if (need == 0) return WC_ERR_INVALID_ARG;  // unknown dtype
  if (need > WC_NOALLOC_SCRATCH_BYTES) return WC_ERR_CAPACITY;  // more values than the array serves
  int32_t err = WC_OK;
  void *scratch = scratch_address(&err);
  if (err != WC_OK) return err;
  // The encode pipeline clears the counters and histogram it keeps in scratch
  // at the start of every call, so what a previous call left there does not
  // matter and nothing else needs clearing here.
  return wc_encode(d_in, n, dtype, d_out, out_cap, scratch, WC_NOALLOC_SCRATCH_BYTES, d_out_size,
                   stream);
}
