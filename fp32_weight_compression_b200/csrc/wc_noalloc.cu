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
#include <cuda.h>

#include <mutex>

#include "wc.h"
#include "wc_format.cuh"

namespace {

// The library-held scratch (see the header comment of wc_encode_noalloc).
static __device__ __align__(256) uint8_t g_noalloc_scratch[WC_NOALLOC_SCRATCH_BYTES];

// The most values the array serves: the largest whole number of chunks whose
// wc_scratch_bytes fits WC_NOALLOC_SCRATCH_BYTES (the same for every dtype).
uint64_t max_values() {
  uint64_t nc = 0;
  while (wc::scratch_win_offset(nc + 1) + (nc + 1) * wc::kWin <= WC_NOALLOC_SCRATCH_BYTES) nc++;
  return nc * wc::kChunk;
}

}  // namespace

namespace wc {

// Identity of the CUDA context current on this thread (0 if there is none or
// the driver cannot say).  A device's array lives in the module loaded into
// that device's context; if the context is destroyed and created again (a
// cudaDeviceReset, a primary-context release), the array may move, so a
// cached address is only reused inside the context it was looked up in.
// The driver calls are reached through the runtime's entry-point lookup, so
// the library does not link the driver library itself.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext *);
  using GetId = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace wc

namespace {

// Device address of g_noalloc_scratch on the current device, looked up with
// that device current (in host code the symbol's name is only a host-side
// stand-in, never a device address) and cached per device together with the
// context it belongs to.
void *scratch_address(int32_t *err) {
  struct Entry {
    void *addr = nullptr;
    unsigned long long ctx = 0;
  };
  static std::mutex mu;
  static Entry cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *err = WC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  Entry &c = cache[dev];
  const unsigned long long ctx = wc::current_context_id();
  if (c.addr == nullptr || ctx == 0 || c.ctx != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *err = WC_ERR_CUDA;
      return nullptr;
    }
    c.addr = p;
    c.ctx = wc::current_context_id();  // the lookup made the device's context current
  }
  *err = WC_OK;
  return c.addr;
}

}  // namespace

extern "C" WC_API int32_t wc_encode_noalloc(const void *d_in, uint64_t n, int32_t dtype, void *d_out,
                                            uint64_t out_cap, uint64_t *d_out_size, void *stream) {
  if (wc_scratch_bytes(0, dtype) == 0) return WC_ERR_INVALID_ARG;  // unknown dtype
  static const uint64_t kMaxValues = max_values();
  if (n > kMaxValues) return WC_ERR_CAPACITY;  // more values than the array serves
  int32_t err = WC_OK;
  void *scratch = scratch_address(&err);
  if (err != WC_OK) return err;
  // The encode pipeline clears the counters and histogram it keeps in scratch
  // at the start of every call, so what a previous call left there does not
  // matter and nothing else needs clearing here.
  return wc_encode(d_in, n, dtype, d_out, out_cap, scratch, WC_NOALLOC_SCRATCH_BYTES, d_out_size,
                   stream);
}
