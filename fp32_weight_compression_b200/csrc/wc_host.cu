// wc_host.cu -- encode and decode of host-resident tensors through the device
// in windows ("seedpack 0.2.0 -> 0.2.2", README: a BF16 model larger than the
// GPU's memory is handled in groups of tensors of roughly a gigabyte and
// unpacked on the GPU one tensor after another).
//
// The caller's device workspace is cut into K slots (K = 3 when the largest
// item allows it, else 2, else 1).  Consecutive items are grouped into
// windows that fit one slot, and window w uses slot w mod K.  Three streams
// form a pipeline: copies host -> device on stream_in, the batched kernels on
// stream_compute, copies device -> host on stream_out, ordered by events:
//   in(w)  waits for out(w - K)   (the slot's previous window has left)
//   compute(w) waits for in(w)
//   out(w) waits for compute(w)
// so that with K = 3 the copies in both directions and the kernels of three
// consecutive windows overlap.  Encoding needs each container's size on the
// host before its copy back: the host reads the sizes of window w - 1 (on a
// stream of its own, so the read waits for the encode of w - 1 and nothing
// else) after it has queued window w, so the device never waits for the host.
#include <cstring>
#include <vector>

#include "wc.h"
#include "wc_format.cuh"

namespace {

inline uint64_t r256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

uint64_t elem_bytes(int32_t dt) { return wc::dtype_bytes(dt); }

bool dtype_ok(int32_t dt) {
  return dt == WC_BF16 || dt == WC_FP32 || dt == WC_FP16 || dt == WC_FP8E4M3 || dt == WC_FP8E5M2;
}

constexpr uint64_t kWindowReserve = 256;  // per window: the rounding of its size array

// Workspace bytes ahead of the slots: one int32 status word per item.
uint64_t head_bytes(uint32_t count) { return r256(4 * uint64_t(count)); }

struct Events {
  std::vector<cudaEvent_t> ev;
  bool ok = true;
  explicit Events(int n) : ev(n, nullptr) {
    for (auto &e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) ok = false;
  }
  ~Events() {
    for (auto &e : ev)
      if (e) cudaEventDestroy(e);
  }
};

// A non-blocking stream owned by one call.
struct OwnStream {
  cudaStream_t s = nullptr;
  bool ok = false;
  OwnStream() { ok = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess; }
  ~OwnStream() {
    if (s) cudaStreamDestroy(s);
  }
};

int32_t fail(cudaError_t e) { return e == cudaSuccess ? WC_OK : WC_ERR_CUDA; }

}  // namespace

extern "C" {

uint64_t wc_host_encode_footprint(uint64_t n, int32_t dtype) {
  const uint64_t bound = wc_encode_bound(n, dtype);
  if (bound == 0) return 0;
  return r256(n * elem_bytes(dtype)) + r256(bound) + r256(wc_scratch_bytes(n, dtype)) + 8;
}

uint64_t wc_host_decode_footprint(uint64_t cont_bytes, uint64_t n, int32_t dtype) {
  if (!dtype_ok(dtype)) return 0;
  return r256(cont_bytes) + r256(n * elem_bytes(dtype));
}

int32_t wc_host_plan(const uint64_t *footprints, uint32_t count, uint64_t slot_area,
                     uint64_t window_bytes, uint32_t *slots, uint32_t *window_end,
                     uint32_t *n_windows) {
  if (slots == nullptr || n_windows == nullptr) return WC_ERR_INVALID_ARG;
  *slots = 0;
  *n_windows = 0;
  if (count == 0) return WC_OK;
  if (footprints == nullptr || window_end == nullptr) return WC_ERR_INVALID_ARG;
  uint64_t big = 0;
  for (uint32_t i = 0; i < count; i++) {
    if (footprints[i] == 0) return WC_ERR_INVALID_ARG;
    big = footprints[i] > big ? footprints[i] : big;
  }
  uint32_t k = 3;
  while (k > 0 && (slot_area / k) / 256 * 256 < big + kWindowReserve) k--;
  if (k == 0) return WC_ERR_CAPACITY;
  const uint64_t slot = (slot_area / k) / 256 * 256;
  const uint64_t cap = window_bytes && window_bytes < slot ? window_bytes : slot;
  uint32_t w = 0;
  uint64_t used = kWindowReserve;
  for (uint32_t i = 0; i < count; i++) {
    // close the window before item i (an item alone may exceed window_bytes)
    if (used > kWindowReserve && used + footprints[i] > cap) {
      window_end[w++] = i;
      used = kWindowReserve;
    }
    used += footprints[i];
  }
  window_end[w++] = count;
  *slots = k;
  *n_windows = w;
  return WC_OK;
}

int32_t wc_encode_host(const wc_host_encode_item *items, uint32_t count, void *d_work,
                       uint64_t work_cap, uint64_t window_bytes, void *stream_in,
                       void *stream_compute, void *stream_out) {
  if (count == 0) return WC_OK;
  if (items == nullptr || d_work == nullptr || (reinterpret_cast<uintptr_t>(d_work) & 255))
    return WC_ERR_INVALID_ARG;
  std::vector<uint64_t> fp(count);
  for (uint32_t i = 0; i < count; i++) {
    const wc_host_encode_item &it = items[i];
    if (!dtype_ok(it.dtype) || it.reserved != 0) return WC_ERR_INVALID_ARG;
    if ((it.n > 0 && it.h_in == nullptr) || it.h_out == nullptr || it.h_out_size == nullptr)
      return WC_ERR_INVALID_ARG;
    fp[i] = wc_host_encode_footprint(it.n, it.dtype);
    if (fp[i] == 0) return WC_ERR_UNSUPPORTED;
    if (it.h_out_cap < wc_encode_bound(it.n, it.dtype)) return WC_ERR_CAPACITY;
  }
  const uint64_t head = head_bytes(count);
  if (work_cap <= head) return WC_ERR_CAPACITY;
  uint32_t K = 0, W = 0;
  std::vector<uint32_t> wend(count);
  int32_t st = wc_host_plan(fp.data(), count, work_cap - head, window_bytes, &K, wend.data(), &W);
  if (st != WC_OK) return st;
  const uint64_t slot_bytes = ((work_cap - head) / K) / 256 * 256;
  uint8_t *work = static_cast<uint8_t *>(d_work);
  cudaStream_t s_in = static_cast<cudaStream_t>(stream_in);
  cudaStream_t s_cp = static_cast<cudaStream_t>(stream_compute);
  cudaStream_t s_out = static_cast<cudaStream_t>(stream_out);
  Events E(3 * K);  // [0, K) copied in, [K, 2K) encoded, [2K, 3K) copied out
  OwnStream szs;    // size read-back, so that it waits for nothing but its window
  if (!E.ok || !szs.ok) return WC_ERR_CUDA;

  // device addresses of window w's items
  std::vector<wc_encode_item> di(count);
  std::vector<uint64_t> sizes(count);
  auto lay_out = [&](uint32_t w) {
    const uint32_t b = w ? wend[w - 1] : 0, e = wend[w];
    uint8_t *p = work + head + uint64_t(w % K) * slot_bytes;
    uint64_t *sz = reinterpret_cast<uint64_t *>(p);
    p += r256(8 * uint64_t(e - b));
    for (uint32_t i = b; i < e; i++) {
      const wc_host_encode_item &it = items[i];
      wc_encode_item &d = di[i];
      d.in = p;
      p += r256(it.n * elem_bytes(it.dtype));
      d.n = it.n;
      d.dtype = it.dtype;
      d.reserved = 0;
      d.out = p;
      d.out_cap = wc_encode_bound(it.n, it.dtype);
      p += r256(d.out_cap);
      d.scratch = p;
      d.scratch_cap = wc_scratch_bytes(it.n, it.dtype);
      p += r256(d.scratch_cap);
      d.out_size = sz + (i - b);
    }
  };
  // Copy window v's containers back.  The host waits for window v's encode
  // only (its sizes come back on a stream of their own), not for the copies
  // of earlier windows still queued on stream_out.
  auto finish = [&](uint32_t v) -> int32_t {
    const uint32_t b = v ? wend[v - 1] : 0, e = wend[v];
    const uint32_t s = v % K;
    cudaError_t ce = cudaStreamWaitEvent(szs.s, E.ev[K + s], 0);
    if (ce == cudaSuccess)  // pageable destination: returns once the copy is done
      ce = cudaMemcpyAsync(sizes.data() + b, di[b].out_size, 8 * uint64_t(e - b),
                           cudaMemcpyDeviceToHost, szs.s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(szs.s);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s_out, E.ev[K + s], 0);
    if (ce != cudaSuccess) return fail(ce);
    for (uint32_t i = b; i < e; i++) {
      if (sizes[i] > items[i].h_out_cap) return WC_ERR_CAPACITY;
      *items[i].h_out_size = sizes[i];
      if (sizes[i] && (ce = cudaMemcpyAsync(items[i].h_out, di[i].out, sizes[i],
                                            cudaMemcpyDeviceToHost, s_out)) != cudaSuccess)
        return fail(ce);
    }
    return fail(cudaEventRecord(E.ev[2 * K + s], s_out));
  };

  for (uint32_t w = 0; w < W && st == WC_OK; w++) {
    const uint32_t b = w ? wend[w - 1] : 0, e = wend[w];
    const uint32_t s = w % K;
    if (K == 1 && w >= 1 && (st = finish(w - 1)) != WC_OK) break;
    cudaError_t ce = cudaSuccess;
    if (w >= K) ce = cudaStreamWaitEvent(s_in, E.ev[2 * K + s], 0);
    lay_out(w);
    for (uint32_t i = b; i < e && ce == cudaSuccess; i++) {
      const uint64_t bytes = items[i].n * elem_bytes(items[i].dtype);
      if (bytes) ce = cudaMemcpyAsync(const_cast<void *>(di[i].in), items[i].h_in, bytes,
                                      cudaMemcpyHostToDevice, s_in);
    }
    if (ce == cudaSuccess) ce = cudaEventRecord(E.ev[s], s_in);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s_cp, E.ev[s], 0);
    if (ce != cudaSuccess) { st = fail(ce); break; }
    if ((st = wc_encode_batch(di.data() + b, e - b, s_cp)) != WC_OK) break;
    if ((ce = cudaEventRecord(E.ev[K + s], s_cp)) != cudaSuccess) { st = fail(ce); break; }
    if (K > 1 && w >= 1) st = finish(w - 1);
  }
  if (st == WC_OK) st = finish(W - 1);
  // leave nothing of this call in flight, whatever happened
  const cudaError_t a = cudaStreamSynchronize(s_in), c = cudaStreamSynchronize(s_cp),
                    o = cudaStreamSynchronize(s_out);
  if (st == WC_OK) st = fail(a != cudaSuccess ? a : (c != cudaSuccess ? c : o));
  return st;
}

int32_t wc_decode_host(const wc_host_decode_item *items, uint32_t count, void *d_work,
                       uint64_t work_cap, uint64_t window_bytes, void *stream_in,
                       void *stream_compute, void *stream_out, int32_t *h_status) {
  if (h_status == nullptr) return WC_ERR_INVALID_ARG;
  *h_status = WC_OK;
  if (count == 0) return WC_OK;
  if (items == nullptr || d_work == nullptr || (reinterpret_cast<uintptr_t>(d_work) & 255))
    return WC_ERR_INVALID_ARG;
  std::vector<uint64_t> fp(count), out_bytes(count);
  for (uint32_t i = 0; i < count; i++) {
    const wc_host_decode_item &it = items[i];
    if (it.h_cont == nullptr) return WC_ERR_INVALID_ARG;
    uint64_t n = 0, nc = 0;
    int32_t dt = 0;
    const int32_t hs = wc_read_header(it.h_cont, it.cont_bytes, &n, &dt, &nc);
    if (hs != WC_OK) return hs;
    out_bytes[i] = n * elem_bytes(dt);
    if (out_bytes[i] > it.out_cap || (out_bytes[i] > 0 && it.h_out == nullptr))
      return WC_ERR_CAPACITY;
    fp[i] = wc_host_decode_footprint(it.cont_bytes, n, dt);
  }
  const uint64_t head = head_bytes(count);
  if (work_cap <= head) return WC_ERR_CAPACITY;
  uint32_t K = 0, W = 0;
  std::vector<uint32_t> wend(count);
  int32_t st = wc_host_plan(fp.data(), count, work_cap - head, window_bytes, &K, wend.data(), &W);
  if (st != WC_OK) return st;
  const uint64_t slot_bytes = ((work_cap - head) / K) / 256 * 256;
  uint8_t *work = static_cast<uint8_t *>(d_work);
  int32_t *d_status = reinterpret_cast<int32_t *>(work);
  cudaStream_t s_in = static_cast<cudaStream_t>(stream_in);
  cudaStream_t s_cp = static_cast<cudaStream_t>(stream_compute);
  cudaStream_t s_out = static_cast<cudaStream_t>(stream_out);
  Events E(3 * K);  // [0, K) copied in, [K, 2K) decoded, [2K, 3K) copied out
  if (!E.ok) return WC_ERR_CUDA;
  std::vector<wc_decode_item> di(count);

  for (uint32_t w = 0; w < W && st == WC_OK; w++) {
    const uint32_t b = w ? wend[w - 1] : 0, e = wend[w];
    const uint32_t s = w % K;
    uint8_t *p = work + head + uint64_t(s) * slot_bytes + kWindowReserve;
    for (uint32_t i = b; i < e; i++) {
      di[i].cont = p;
      di[i].cont_bytes = items[i].cont_bytes;
      p += r256(items[i].cont_bytes);
      di[i].out = p;
      di[i].out_cap = out_bytes[i];
      p += r256(out_bytes[i]);
    }
    cudaError_t ce = cudaSuccess;
    if (w >= K) ce = cudaStreamWaitEvent(s_in, E.ev[2 * K + s], 0);
    for (uint32_t i = b; i < e && ce == cudaSuccess; i++)
      ce = cudaMemcpyAsync(const_cast<void *>(di[i].cont), items[i].h_cont, items[i].cont_bytes,
                           cudaMemcpyHostToDevice, s_in);
    if (ce == cudaSuccess) ce = cudaEventRecord(E.ev[s], s_in);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s_cp, E.ev[s], 0);
    if (ce != cudaSuccess) { st = fail(ce); break; }
    if ((st = wc_decode_batch(di.data() + b, e - b, d_status + w, s_cp)) != WC_OK) break;
    ce = cudaEventRecord(E.ev[K + s], s_cp);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s_out, E.ev[K + s], 0);
    for (uint32_t i = b; i < e && ce == cudaSuccess; i++)
      if (out_bytes[i]) ce = cudaMemcpyAsync(items[i].h_out, di[i].out, out_bytes[i],
                                             cudaMemcpyDeviceToHost, s_out);
    if (ce == cudaSuccess) ce = cudaEventRecord(E.ev[2 * K + s], s_out);
    if (ce != cudaSuccess) st = fail(ce);
  }
  const cudaError_t a = cudaStreamSynchronize(s_in), c = cudaStreamSynchronize(s_cp),
                    o = cudaStreamSynchronize(s_out);
  if (st == WC_OK) st = fail(a != cudaSuccess ? a : (c != cudaSuccess ? c : o));
  if (st == WC_OK) {
    std::vector<int32_t> ws(W);
    cudaError_t ce = cudaMemcpyAsync(ws.data(), d_status, 4 * uint64_t(W), cudaMemcpyDeviceToHost, s_out);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s_out);
    if (ce != cudaSuccess) return fail(ce);
    for (uint32_t w = 0; w < W; w++)
      if (ws[w] != WC_OK) { *h_status = ws[w]; break; }
  }
  return st;
}

}  // extern "C"
