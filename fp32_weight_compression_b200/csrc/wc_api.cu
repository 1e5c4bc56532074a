// wc_api.cu -- the C ABI (include/wc.h): argument checks, batching of tensors
// into launches, and the kernel launch sequence.
//
// Encode, per launch of up to kMaxItems tensors (all on `stream`):
//   k_prep     header fields + scratch counters            (1 block / tensor)
//   k_hist     coded-byte histogram -> 12-bit table        (1 block / 4 chunks)
//   k_coder    raw planes + rANS per chunk + offset scan   (1 warp / 2 chunks)
//   k_compact  payloads into the exponent section          (1 block / chunk)
// Decode, per launch of up to kMaxItems containers:
//   k_decode   persistent grid, one warp per 2 chunks
// Block checksums (wc_crc32_blocks):
//   k_crc32    persistent grid, one block of the buffer per CTA at a time
#include <cstdio>
#include <cstring>
#include <mutex>

#include "wc.h"
#include "wc_format.cuh"

namespace wc {
// block checksums (k_crc.cu)
cudaError_t launch_crc32(const uint8_t *buf, uint64_t bytes, uint64_t block_bytes, uint32_t *crc,
                         int grid, cudaStream_t s);
int crc_blocks_per_sm();
}  // namespace wc

namespace {

thread_local char g_last_error[256] = "";

int32_t cuda_fail(cudaError_t e, const char *where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return WC_ERR_CUDA;
}

constexpr uint64_t kMaxN = uint64_t(1) << 44;


bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool dtype_ok(int32_t dt) {
  return dt == WC_BF16 || dt == WC_FP32 || dt == WC_FP16 || dt == WC_FP8E4M3 || dt == WC_FP8E5M2;
}

struct DeviceInfo {
  int sms = 0;
  int dec_blocks_per_sm = 0;
  int crc_blocks_per_sm = 0;
  cudaError_t crc_err = cudaSuccess;
  unsigned long long ctx = 0;  // the context the kernels' attributes were set in
};

DeviceInfo device_info(int32_t *err) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *err = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cudaGetDevice");
    return DeviceInfo{};
  }
  std::lock_guard<std::mutex> lock(mu);
  // once per device, and again in a context created afresh (after a
  // cudaDeviceReset the kernels' shared-memory attributes must be set again)
  const unsigned long long ctx = wc::current_context_id();
  if (cache[dev].sms == 0 || (ctx != 0 && cache[dev].ctx != ctx)) {
    cache[dev] = DeviceInfo{};
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
      *err = cuda_fail(e, "cudaDeviceGetAttribute");
      return DeviceInfo{};
    }
    const int nb = wc::decode_blocks_per_sm();
    if (nb <= 0) {
      *err = cuda_fail(cudaGetLastError(), "decoder set-up");
      return DeviceInfo{};
    }

    // the checksum kernel's set-up failing leaves the codec usable
    cache[dev].crc_blocks_per_sm = wc::crc_blocks_per_sm();
    if (cache[dev].crc_blocks_per_sm <= 0) cache[dev].crc_err = cudaGetLastError();
    cache[dev].dec_blocks_per_sm = nb;
    cache[dev].sms = sms;
    cache[dev].ctx = wc::current_context_id();  // the set-up made the device's context current
  }
  *err = WC_OK;
  return cache[dev];
}

}  // namespace

extern "C" {

uint64_t wc_encode_bound(uint64_t n, int32_t dtype) {
  if (!dtype_ok(dtype) || n > kMaxN) return 0;
  const wc::Layout L = wc::make_layout(n, dtype);
  uint64_t exp = 0;
  if (L.nc) exp = (L.nc - 1) * uint64_t(wc::kChunk) + wc::round16(wc::chunk_nsym(n, L.nc - 1));
  return L.off_exp + exp;
}

uint64_t wc_scratch_bytes(uint64_t n, int32_t dtype) {
  if (!dtype_ok(dtype) || n > kMaxN) return 0;
  const uint64_t nc = wc::num_chunks(n);
  return wc::scratch_win_offset(nc) + nc * wc::kWin;
}

int32_t wc_crc32_blocks(const void *d_buf, uint64_t bytes, uint64_t block_bytes, uint32_t *d_crc,
                        void *stream) {
  if (block_bytes == 0 || block_bytes % 8192 != 0 || block_bytes > (uint64_t(1) << 30))
    return WC_ERR_INVALID_ARG;
  if (bytes == 0) return WC_OK;
  if (d_buf == nullptr || d_crc == nullptr || !aligned(d_buf, 16) || !aligned(d_crc, 4))
    return WC_ERR_INVALID_ARG;
  int32_t err = WC_OK;
  const DeviceInfo di = device_info(&err);
  if (err != WC_OK) return err;
  if (di.crc_blocks_per_sm <= 0)
    return cuda_fail(di.crc_err == cudaSuccess ? cudaErrorInvalidConfiguration : di.crc_err,
                     "k_crc32 set-up");
  const uint64_t nblocks = (bytes + block_bytes - 1) / block_bytes;
  const uint64_t cap = uint64_t(di.sms) * uint64_t(di.crc_blocks_per_sm);
  const int grid = int(nblocks < cap ? nblocks : cap);
  const cudaError_t e = wc::launch_crc32(static_cast<const uint8_t *>(d_buf), bytes, block_bytes,
                                         d_crc, grid, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WC_OK : cuda_fail(e, "k_crc32 launch");
}

const char *wc_status_string(int32_t st) {
  switch (st) {
    case WC_OK: return "WC_OK";
    case WC_ERR_INVALID_ARG: return "WC_ERR_INVALID_ARG";
    case WC_ERR_CAPACITY: return "WC_ERR_CAPACITY";
    case WC_ERR_CUDA: return "WC_ERR_CUDA";
    case WC_ERR_CORRUPT: return "WC_ERR_CORRUPT";
    case WC_ERR_UNSUPPORTED: return "WC_ERR_UNSUPPORTED";
    case WC_ERR_TIMEOUT: return "WC_ERR_TIMEOUT";
    default: return "WC_ERR_UNKNOWN";
  }
}

const char *wc_last_error(void) { return g_last_error; }

int32_t wc_encode_batch(const wc_encode_item *items, uint32_t count, void *stream) {
  if (count == 0) return WC_OK;
  if (items == nullptr) return WC_ERR_INVALID_ARG;
  for (uint32_t i = 0; i < count; i++) {
    const wc_encode_item &it = items[i];
    if (!dtype_ok(it.dtype) || it.reserved != 0) return WC_ERR_INVALID_ARG;
    if (it.n > kMaxN) return WC_ERR_UNSUPPORTED;
    if (it.n > 0 && (it.in == nullptr || !aligned(it.in, 16))) return WC_ERR_INVALID_ARG;
    if (it.out == nullptr || !aligned(it.out, 16) || it.out_size == nullptr || !aligned(it.out_size, 8))
      return WC_ERR_INVALID_ARG;
    if (it.scratch == nullptr || !aligned(it.scratch, 256)) return WC_ERR_INVALID_ARG;
    if (it.out_cap < wc_encode_bound(it.n, it.dtype)) return WC_ERR_CAPACITY;
    if (it.scratch_cap < wc_scratch_bytes(it.n, it.dtype)) return WC_ERR_CAPACITY;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local wc::EncParams P;  // ~14 KiB: kept off the stack
  for (uint32_t b0 = 0; b0 < count; b0 += wc::kMaxItems) {
    const uint32_t cnt = count - b0 < wc::kMaxItems ? count - b0 : wc::kMaxItems;
    memset(&P, 0, sizeof(P));
    P.count = cnt;
    uint64_t chunks = 0, blocks = 0, hblocks = 0;
    for (uint32_t i = 0; i < cnt; i++) {
      const wc_encode_item &src = items[b0 + i];
      wc::EncItem &d = P.items[i];
      d.in = static_cast<const uint8_t *>(src.in);
      d.out = static_cast<uint8_t *>(src.out);
      d.scratch = static_cast<uint8_t *>(src.scratch);
      d.out_size = src.out_size;
      d.n = src.n;
      d.dtype = uint32_t(src.dtype);
      d.chunk_base = uint32_t(chunks);
      d.block_base = uint32_t(blocks);
      d.hist_base = uint32_t(hblocks);
      const uint64_t nc = wc::num_chunks(src.n);
      chunks += nc;
      blocks += (nc + wc::kCoderChunks - 1) / wc::kCoderChunks;
      hblocks += (nc + wc::kHistChunks - 1) / wc::kHistChunks;
      if (chunks >= (uint64_t(1) << 31)) return WC_ERR_UNSUPPORTED;
    }
    P.total_chunks = uint32_t(chunks);
    P.total_coder_blocks = uint32_t(blocks);
    P.total_hist_blocks = uint32_t(hblocks);
    cudaError_t e;
    if ((e = wc::launch_prep(P, s)) != cudaSuccess) return cuda_fail(e, "k_prep");
    if ((e = wc::launch_hist(P, s)) != cudaSuccess) return cuda_fail(e, "k_hist");
    if ((e = wc::launch_coder(P, s)) != cudaSuccess) return cuda_fail(e, "k_coder");
    if ((e = wc::launch_compact(P, s)) != cudaSuccess) return cuda_fail(e, "k_compact");
  }
  return WC_OK;
}

int32_t wc_encode(const void *d_in, uint64_t n, int32_t dtype, void *d_out, uint64_t out_cap,
                  void *d_scratch, uint64_t scratch_cap, uint64_t *d_out_size, void *stream) {
  wc_encode_item it;
  it.in = d_in;
  it.n = n;
  it.dtype = dtype;
  it.reserved = 0;
  it.out = d_out;
  it.out_cap = out_cap;
  it.scratch = d_scratch;
  it.scratch_cap = scratch_cap;
  it.out_size = d_out_size;
  return wc_encode_batch(&it, 1, stream);
}

static int32_t check_dec_item(const wc::DecItem &it) {
  if (it.cont == nullptr || !aligned(it.cont, 16)) return WC_ERR_INVALID_ARG;
  if (it.out_cap > 0 && (it.out == nullptr || !aligned(it.out, 16))) return WC_ERR_INVALID_ARG;
  return WC_OK;
}

// Queue the decode of `count` (<= kMaxItems) already-validated items.  With
// clear_status the status word is cleared first (stream-ordered).
static int32_t decode_slice(const wc::DecItem *items, uint32_t count, int32_t *d_status,
                            bool clear_status, cudaStream_t s) {
  int32_t err = WC_OK;
  const DeviceInfo info = device_info(&err);
  if (err != WC_OK) return err;
  cudaError_t e;
  if (clear_status && (e = cudaMemsetAsync(d_status, 0, sizeof(int32_t), s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync(status)");
  if (count == 0) return WC_OK;
  static thread_local wc::DecParams P;  // ~12 KiB: kept off the stack
  memset(&P, 0, sizeof(P));
  P.count = count;
  P.status = d_status;
  for (uint32_t i = 0; i < count; i++) P.items[i] = items[i];
  if ((e = wc::launch_decode(P, info.sms * info.dec_blocks_per_sm, s)) != cudaSuccess)
    return cuda_fail(e, "k_decode");
  return WC_OK;
}

int32_t wc_decode_batch(const wc_decode_item *items, uint32_t count, int32_t *d_status,
                        void *stream) {
  if ((count > 0 && items == nullptr) || d_status == nullptr || !aligned(d_status, 4))
    return WC_ERR_INVALID_ARG;
  static thread_local wc::DecItem tmp[wc::kMaxItems];
  auto convert = [&](uint32_t i) {
    wc::DecItem d;
    d.cont = static_cast<const uint8_t *>(items[i].cont);
    d.cont_bytes = items[i].cont_bytes;
    d.out = static_cast<uint8_t *>(items[i].out);
    d.out_cap = items[i].out_cap;
    d.chunk_first = 0;
    d.chunk_count = ~uint64_t(0);
    return d;
  };
  for (uint32_t i = 0; i < count; i++) {
    const int32_t st = check_dec_item(convert(i));
    if (st != WC_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (count == 0) return decode_slice(tmp, 0, d_status, true, s);
  for (uint32_t b0 = 0; b0 < count; b0 += wc::kMaxItems) {
    const uint32_t cnt = count - b0 < wc::kMaxItems ? count - b0 : wc::kMaxItems;
    for (uint32_t i = 0; i < cnt; i++) tmp[i] = convert(b0 + i);
    const int32_t st = decode_slice(tmp, cnt, d_status, b0 == 0, s);
    if (st != WC_OK) return st;
  }
  return WC_OK;
}

static int32_t decode_one(const wc::DecItem &it, int32_t *d_status, void *stream) {
  if (d_status == nullptr || !aligned(d_status, 4)) return WC_ERR_INVALID_ARG;
  const int32_t st = check_dec_item(it);
  if (st != WC_OK) return st;
  return decode_slice(&it, 1, d_status, true, static_cast<cudaStream_t>(stream));
}

int32_t wc_decode(const void *d_cont, uint64_t cont_bytes, void *d_out, uint64_t out_cap,
                  int32_t *d_status, void *stream) {
  wc::DecItem it;
  it.cont = static_cast<const uint8_t *>(d_cont);
  it.cont_bytes = cont_bytes;
  it.out = static_cast<uint8_t *>(d_out);
  it.out_cap = out_cap;
  it.chunk_first = 0;
  it.chunk_count = ~uint64_t(0);
  return decode_one(it, d_status, stream);
}

int32_t wc_decode_chunk(const void *d_cont, uint64_t cont_bytes, uint64_t k, void *d_out,
                        uint64_t out_cap, int32_t *d_status, void *stream) {
  wc::DecItem it;
  it.cont = static_cast<const uint8_t *>(d_cont);
  it.cont_bytes = cont_bytes;
  it.out = static_cast<uint8_t *>(d_out);
  it.out_cap = out_cap;
  it.chunk_first = k;
  it.chunk_count = 1;
  return decode_one(it, d_status, stream);
}

int32_t wc_read_header(const void *h_cont, uint64_t bytes, uint64_t *n, int32_t *dtype,
                       uint64_t *nchunks) {
  if (h_cont == nullptr || n == nullptr || dtype == nullptr || nchunks == nullptr)
    return WC_ERR_INVALID_ARG;
  if (bytes < wc::kHeaderBytes) return WC_ERR_CORRUPT;
  const uint8_t *c = static_cast<const uint8_t *>(h_cont);
  auto u16 = [&](uint64_t o) { return uint32_t(c[o]) | uint32_t(c[o + 1]) << 8; };
  auto u32 = [&](uint64_t o) { return u16(o) | u16(o + 2) << 16; };
  auto u64 = [&](uint64_t o) { return uint64_t(u32(o)) | uint64_t(u32(o + 4)) << 32; };
  if (memcmp(c, "WCZ1", 4) != 0 || u16(4) != wc::kVersion || c[7] != wc::kLanes) return WC_ERR_CORRUPT;
  const int32_t dt = c[6];
  if (!dtype_ok(dt)) return WC_ERR_CORRUPT;
  const uint64_t nn = u64(8);
  if (nn > kMaxN) return WC_ERR_CORRUPT;
  if (u32(16) != wc::kChunk || u32(24) != wc::kProbBits || u32(28) != 0) return WC_ERR_CORRUPT;
  const wc::Layout L = wc::make_layout(nn, dt);
  if (u32(20) != uint32_t(L.nc) || u64(32) != L.off_raw || u64(40) != L.off_exp) return WC_ERR_CORRUPT;
  if (u64(56) != L.off_exp + u64(48)) return WC_ERR_CORRUPT;
  if (bytes >= L.off_raw) {
    // offset table present: check it too
    uint32_t sum = 0;
    for (int s = 0; s < 256; s++) sum += u16(wc::kFreqOffset + 2 * s);
    if (nn == 0 ? sum != 0 : sum != wc::kProbScale) return WC_ERR_CORRUPT;
    if (u64(L.off_chunk_off) != 0) return WC_ERR_CORRUPT;
    for (uint64_t k = 0; k < L.nc; k++) {
      const uint32_t nsym = wc::chunk_nsym(nn, k);
      const uint32_t len = u32(L.off_chunk_len + 4 * k);
      const bool raw = len == nsym;
      const bool coded = len >= wc::kStateBytes && len < nsym && (len & 1u) == 0;
      if (!raw && !coded) return WC_ERR_CORRUPT;
      if (u64(L.off_chunk_off + 8 * (k + 1)) != u64(L.off_chunk_off + 8 * k) + wc::round16(len))
        return WC_ERR_CORRUPT;
    }
    if (u64(L.off_chunk_off + 8 * L.nc) != u64(48)) return WC_ERR_CORRUPT;
  }
  *n = nn;
  *dtype = dt;
  *nchunks = L.nc;
  return WC_OK;
}

int32_t wc_chunk_ranges(const void *h_prefix, uint64_t prefix_bytes, uint64_t k, uint64_t *ranges,
                        uint32_t *count) {
  if (h_prefix == nullptr || ranges == nullptr || count == nullptr) return WC_ERR_INVALID_ARG;
  uint64_t n = 0, nc = 0;
  int32_t dt = 0;
  const int32_t st = wc_read_header(h_prefix, prefix_bytes, &n, &dt, &nc);
  if (st != WC_OK) return st;
  const wc::Layout L = wc::make_layout(n, dt);
  // with the whole prefix present, wc_read_header has checked every table entry
  if (prefix_bytes < L.off_raw) return WC_ERR_CAPACITY;
  if (k >= nc) return WC_ERR_INVALID_ARG;
  const uint8_t *c = static_cast<const uint8_t *>(h_prefix);
  uint64_t choff = 0;
  uint32_t len = 0;
  memcpy(&choff, c + L.off_chunk_off + 8 * k, 8);
  memcpy(&len, c + L.off_chunk_len + 4 * k, 4);
  const uint64_t first = k * wc::kChunk, nsym = wc::chunk_nsym(n, k);
  uint32_t m = 0;
  auto put = [&](uint64_t off, uint64_t bytes) {
    ranges[2 * m] = off;
    ranges[2 * m + 1] = bytes;
    m++;
  };
  put(0, L.off_raw);
  if (dt == WC_FP32) {
    put(L.off_raw + first / 8, (nsym + 7) / 8);
    put(L.off_mant + 3 * first, 3 * nsym);
  } else if (wc::is_fp8(dt)) {
    put(L.off_raw + first / 2, (nsym + 1) / 2);
  } else {
    put(L.off_raw + first, nsym);
  }
  put(L.off_exp + choff, wc::round16(len));
  *count = m;
  return WC_OK;
}

}  // extern "C"
