// k_split12_linear.cu -- Y = X W^T with the weights W (N x K, bf16, row-major)
// held as a Split12 container (include/wc_split12.h): the weight tile is
// expanded from the index and low planes straight into the tensor cores'
// shared-memory operand layout and multiplied with tcgen05.mma, accumulating
// in tensor memory, so the weights cross HBM at 12 bits a value ("weight-
// compression" README: Split12 serving, bf16 weights rebuilt on the fly).
//
// Work split.  A CTA owns 128 weight rows (the MMA's M) and a range of K;
// the host splits K across CTAs so that the grid is one wave, and the CTAs
// of one row block add their partial sums into Y (fp32 atomics; Y is zeroed
// first).  Per stage of 64 K-values, in a pipeline without block-wide
// barriers (mbarriers between the roles):
//   * lane 0 of the load warp brings, with TMA, the rows' 64 index nibbles
//     and 64 low bytes each (12 bits a value, as stored) and the tokens' X
//     slice (n_mma rows of 128 bytes, rows past M zero-filled, 128-byte
//     swizzle: the B operand layout) into a ring slot, up to D stages ahead
//     (D = 4, or 3 or 2 where that lets two CTAs share an SM), once the MMAs
//     that read the slot last are done; the slot's mbarrier completes when
//     the bytes have landed;
//   * the 8 expanding warps expand the 128 x 64 values from the ring slot
//     in segments of 16 (8 index bytes + 16 low bytes -> 16 bf16, two
//     16-byte rows of core matrices) into one of two A operand slots (one,
//     in the shape for the largest token counts), patch
//     the tile's exceptions (after a named barrier among them, one thread
//     an exception, its high byte) and arrive on the A slot's mbarrier.  A
//     quarter warp takes 8 consecutive rows of one segment; with the loads'
//     32- and 64-byte swizzles its index and low-byte reads, and its 16-byte
//     stores, each cover 8 distinct bank groups;
//   * lane 0 of the MMA warp waits for the A slot, issues four MMAs (M =
//     128, N = n_mma = M rounded up to 16, K = 16) and commits them to the A
//     slot's and the ring slot's "free" mbarriers, which the expanding warps
//     and the load lane wait on before they reuse either.
// At the end each expanding warp reads its 32 TMEM lanes (rows) and adds them
// into Y.  The tile's exceptions: gathered once per CTA from the container's
// per-chunk lists, or, with the weight's serving plan (wc12_linear_planned,
// wc12_plan.cuh), read from the plan a stage ahead.
//
// Operand layouts (K-major).  A, no swizzle: a core matrix is 8 rows x 16
// bytes stored as 128 contiguous bytes; the two 8-value halves of a K = 16
// slice are 128 bytes apart (leading byte offset) and consecutive 8-row
// groups 256 bytes apart (stride byte offset); a slice is 16 groups = 4 KiB.
// B, 128-byte swizzle: a token's 64 values are one 128-byte row, 8-row
// groups 1024 bytes apart; the K = 16 slice sl starts 32 sl bytes in.
//
// Waits: every mbarrier wait is bounded (and gives up once another thread has
// failed); when one runs out the kernel records
// WC_ERR_TIMEOUT, stops issuing, waits (bounded) for what it issued, frees its
// tensor memory and returns.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "wc.h"
#include "wc12_plan.cuh"
#include "wc_split12.cuh"

namespace wc {
// Identity of the CUDA context current on this thread, 0 if none
// (csrc/wc_noalloc.cu).
unsigned long long current_context_id();
}  // namespace wc

namespace wc12l {

using wc12::kChunk;

constexpr int kExpThreads = 256;         // 8 warps expand; warps 0-3 (TMEM lanes) and 4-7 split the epilogue
constexpr int kMmaWarp = 8;              // lane 0 issues the MMAs
constexpr int kLoadWarp = 9;             // lane 0 issues the TMA loads
constexpr int kThreads = kExpThreads + 64;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr uint32_t kASlice = kBM * 16 * 2;   // bytes of one K = 16 slice of A
constexpr uint32_t kAStage = 4 * kASlice;
constexpr uint32_t kMaxASlots = 2;
constexpr uint32_t kMaxTokens = 256;
constexpr uint32_t kSpinLimit = 1u << 24;
// Without a plan, a CTA's exceptions (its 128 rows, its range of K) are
// gathered once into a shared-memory list of up to kExcCap entries binned by
// stage, {column in the stage, row | high byte << 16}; a CTA with more walks
// its chunks' exception lists at every stage instead.  Either way an exception's value differs from the
// expanded one only in its high byte (the low byte is stored for every value).
constexpr uint32_t kExcCap = 512;
// chunk offsets of a CTA's row block kept in shared memory for the gather
constexpr uint32_t kGatherChunks = 255;

struct Params {
  // tensor maps (tensor-core path): index plane [N rows][K / 2 bytes], box
  // 128 x 32 B, 32-byte swizzle; low plane [N][K bytes], box 128 x 64 B,
  // 64-byte swizzle; X [M][K bf16], box n_mma x 64 values, 128-byte swizzle
  // (rows past M read as zeros)
  CUtensorMap tm_idx, tm_lo, tm_x;
  const uint8_t *w;
  uint64_t w_bytes;
  const uint8_t *plan;  // the container's serving plan (wc12_plan.cuh), or null
  uint64_t plan_bytes;
  const uint16_t *x;  // [M, K]
  float *y;           // [M, N]
  uint32_t M, N, K;
  uint32_t n_mma;     // M rounded up to 16
  uint32_t per_split; // stages per CTA
  uint32_t splits;
  int32_t *status;
};

// Shared memory: the expanded A operand slots (two, or one), then a ring of
// D load slots (the stage's index bytes and low bytes of the 128 rows, as
// stored, and the tokens' X slice already in the B operand layout), the
// mbarriers and, without a plan, the CTA's exception list.  The kernel is
// compiled for four shapes, D = 4, 3 and 2 with two A slots and D = 2 with
// one (constants, so that slot and phase indices are shifts and masks).
constexpr uint32_t kMaxDepth = 4;
// mbarriers (full, slot_free: kMaxDepth each; a_full, a_free: kMaxASlots
// each), the TMEM address, the failure flag and the exception count
constexpr uint32_t kBarBytes = 8 * (2 * kMaxDepth + 2 * kMaxASlots) + 16;
constexpr uint32_t kIdxBytes = kBM * kBK / 2;  // 4 KiB
constexpr uint32_t kLoBytes = kBM * kBK;       // 8 KiB

__host__ __device__ inline uint32_t b_stage_bytes(uint32_t n_mma) { return n_mma * kBK * 2; }
__host__ __device__ inline uint32_t slot_bytes(uint32_t n_mma) { return kIdxBytes + kLoBytes + b_stage_bytes(n_mma); }
// per-stage exception bins: a count (then start) per stage of the CTA
constexpr uint32_t kMaxStagesPerCta = 256;
// the gathered exception list, its bins and cursors, the chunk offsets
constexpr uint32_t kExcBytes = 2 * 8 * kExcCap + 2 * 4 * (kMaxStagesPerCta + 1) + 8 * (kGatherChunks + 1);
__host__ __device__ inline uint32_t smem_bytes(uint32_t n_mma, uint32_t depth, uint32_t aslots, bool plan) {
  return 1024 + aslots * kAStage + depth * slot_bytes(n_mma) + kBarBytes + (plan ? 0u : kExcBytes);
}

__device__ __forceinline__ void report(int32_t *status, int32_t code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// shared-memory matrix descriptor, K-major: leading and stride byte offsets
// lbo and sbo, layout 0 (no swizzle) or 2 (128-byte swizzle)
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(layout) << 61);
}

// instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128, N = n
__device__ __forceinline__ uint32_t instr_desc(uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// true once the phase of the given parity has completed; false after the limit
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t i = 0; i < kSpinLimit; i++) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// byte offset of (row, k) in a stage laid out as K = 16 slices of core matrices
__device__ __forceinline__ uint32_t op_offset(uint32_t row, uint32_t k, uint32_t slice_bytes) {
  return (k >> 4) * slice_bytes + (row >> 3) * 256 + ((k >> 3) & 1) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

// Where TMA puts 16-byte part `part` of row `row` of a plane's box: rows of
// 32 bytes (index plane, 32-byte swizzle: part ^= bit 2 of the row) or 64
// bytes (low plane, 64-byte swizzle: part ^= bits 1-2 of the row).
__device__ __forceinline__ uint32_t idx_gran(uint32_t row, uint32_t part) {
  return row * 32 + ((part ^ ((row >> 2) & 1u)) << 4);
}
__device__ __forceinline__ uint32_t lo_gran(uint32_t row, uint32_t part) {
  return row * 64 + ((part ^ ((row >> 1) & 3u)) << 4);
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// 2-D tile load into this CTA's own shared memory, completing on bar
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier 1 over the expanding threads, returning whether ok holds for
// all of them.
__device__ __forceinline__ bool expanders_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(ok)), "n"(kExpThreads)
      : "memory");
  return r != 0;
}


// A bounded wait that also gives up once another thread of the CTA has
// recorded a failure in *flag.
__device__ __forceinline__ bool mbar_wait_or_flag(uint64_t *bar, uint32_t parity, const volatile int *flag) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t i = 0; i < kSpinLimit; i++) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if (*flag) return false;
  }
  return false;
}

template <uint32_t kDepth, uint32_t kASlots>
__global__ void __launch_bounds__(kThreads, 2) k12_linear(const __grid_constant__ Params p) {
  static_assert(kDepth >= 2 && kDepth <= kMaxDepth, "ring depth");
  static_assert(kASlots >= 1 && kASlots <= kMaxASlots, "A slots");
  extern __shared__ uint8_t dyn[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  uint8_t *a_op = base;                       // kASlots x kAStage
  uint8_t *ring = base + kASlots * kAStage;   // kDepth x slot_bytes
  const uint32_t sb = slot_bytes(p.n_mma);
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + kDepth * sb);  // [kDepth] a slot's loads landed
  uint64_t *slot_free = full + kMaxDepth;                             // [kDepth] its MMAs are done
  uint64_t *a_full = slot_free + kMaxDepth;                              // [kASlots] A slot expanded
  uint64_t *a_free = a_full + kMaxASlots;                             // [kASlots] its MMAs are done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(a_free + kMaxASlots);
  int *flag = reinterpret_cast<int *>(tmem_slot + 1);
  uint32_t *exc_n = tmem_slot + 2;
  // without a plan only:
  uint2 *exc_raw = reinterpret_cast<uint2 *>(reinterpret_cast<uint8_t *>(full) + kBarBytes);  // gathered
  uint2 *exc_bin = exc_raw + kExcCap;                                                        // by stage
  uint32_t *bin = reinterpret_cast<uint32_t *>(exc_bin + kExcCap);                           // per stage
  uint32_t *cur = bin + kMaxStagesPerCta + 1;                                                // cursors
  uint64_t *g_off = reinterpret_cast<uint64_t *>(cur + kMaxStagesPerCta + 1);                 // gather offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool expander = tid < kExpThreads;
  const uint32_t K = p.K, N = p.N;
  const uint32_t n0 = blockIdx.x * kBM;
  const uint32_t split = blockIdx.y;
  const uint32_t total_stages = K / kBK;
  const uint32_t s_begin = split * p.per_split;
  const uint32_t s_end = s_begin + p.per_split < total_stages ? s_begin + p.per_split : total_stages;

  // container header (every CTA checks; CTA (0, 0) reports)
  // (the host refuses containers shorter than 96 bytes, so the header is
  // inside the buffer)
  const uint8_t *w = p.w;
  const uint32_t *h32 = reinterpret_cast<const uint32_t *>(w);
  const uint64_t *h64 = reinterpret_cast<const uint64_t *>(w);
  const uint64_t n = h64[1], ne = h64[3];
  const uint32_t kk = h32[1] >> 24;
  bool ok = h32[0] == wc12::kMagic && (h32[1] & 0xFFFFFFu) == (1u | (1u << 16)) &&
            kk >= 1 && kk <= 16 && n == uint64_t(N) * K && ne <= n && h32[4] == uint32_t(kChunk);
  wc12::Lay L{};
  if (ok) {
    L = wc12::lay(n, ne);
    ok = h32[5] == uint32_t(L.nc) && h64[4] == L.off_idx && h64[5] == L.off_lo && h64[6] == L.off_exc &&
         h64[7] == L.total && L.total <= p.w_bytes;
  }
  if (ok && p.plan != nullptr) {  // a plan built from this container for this N x K
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(p.plan);
    const uint64_t *q64 = reinterpret_cast<const uint64_t *>(p.plan);
    const wc12p::PlanLay P = wc12p::plan_lay(N, K, ne);
    ok = q32[0] == wc12p::kMagic && q32[1] == 1 && q32[2] == N && q32[3] == K && q64[2] == ne &&
         q64[3] == P.buckets && P.total <= p.plan_bytes;
  }
  if (!ok || s_begin >= s_end) {
    if (!ok && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) report(p.status, WC_ERR_CORRUPT);
    return;
  }
  const uint32_t nst = s_end - s_begin;
  const uint4 book = *reinterpret_cast<const uint4 *>(w + wc12::kBookOff);
  const uint64_t *exc_off = reinterpret_cast<const uint64_t *>(w + wc12::kExcOffOff);
  const uint16_t *exc_pos = reinterpret_cast<const uint16_t *>(w + L.off_exc);
  const uint8_t *exc_val = w + L.off_excval;
  const uint64_t c_lo = uint64_t(n0) * K / kChunk, c_hi = (uint64_t(n0 + kBM) * K - 1) / kChunk;

  // stage j's TMA loads into ring slot j % kDepth (the load lane)
  const uint32_t ring_s = smem_u32(ring);
  const uint32_t k_first = s_begin * kBK;
  const uint32_t stage_bytes = kIdxBytes + kLoBytes + b_stage_bytes(p.n_mma);
  auto load_stage = [&](uint32_t j) {
    const uint32_t d = j % kDepth, slot = ring_s + d * sb;
    const int32_t k = int32_t(k_first + j * kBK);
    mbar_expect_tx(&full[d], stage_bytes);
    tma_load_2d(slot, &p.tm_idx, k / 2, int32_t(n0), &full[d]);
    tma_load_2d(slot + kIdxBytes, &p.tm_lo, k, int32_t(n0), &full[d]);
    tma_load_2d(slot + kIdxBytes + kLoBytes, &p.tm_x, k, 0, &full[d]);
  };
  const bool loader = warp == kLoadWarp && lane == 0;

  // tensor memory: n_mma fp32 columns, rounded up to a power of two >= 32
  uint32_t cols = 32;
  while (cols < p.n_mma) cols <<= 1;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (uint32_t d = 0; d < kDepth; d++) {
      mbar_init(&full[d], 1);
      mbar_init(&slot_free[d], 1);
    }
    for (uint32_t d = 0; d < kASlots; d++) {
      mbar_init(&a_full[d], kExpThreads);
      mbar_init(&a_free[d], 1);
    }
    *flag = 0;
    *exc_n = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (p.plan == nullptr)
    for (uint32_t i = tid; i <= nst && i <= kMaxStagesPerCta; i += kThreads) bin[i] = 0;
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // the first kDepth stages' loads are in flight while the exceptions are
  // gathered
  uint32_t loaded = 0;  // load lane: stages whose loads were issued
  if (loader)
    for (; loaded < kDepth && loaded < nst; loaded++) load_stage(loaded);

  // The CTA's exceptions and how they are patched (mode): 0 from a shared
  // list binned by stage (bin[] relative starts), 1 from the plan (bounds
  // and entries read a stage ahead), 2 by walking the chunks' lists at each
  // stage.
  const bool binned = nst <= kMaxStagesPerCta;
  uint32_t mode = 0;
  const uint32_t *plan_start = nullptr, *plan_ent = nullptr;
  if (p.plan != nullptr) {
    // The plan holds the tile's exceptions as one range, by stage: each
    // stage's bounds and a thread's first entry of it are read a stage ahead
    // in the loop, so nothing waits for them before the first stage.
    const wc12p::PlanLay P = wc12p::plan_lay(N, K, ne);
    plan_start = reinterpret_cast<const uint32_t *>(p.plan + wc12p::kStartOff) +
                 uint64_t(blockIdx.x) * (K / kBK) + s_begin;
    plan_ent = reinterpret_cast<const uint32_t *>(p.plan + P.off_ent);
    mode = 1;
  } else {
  // The CTA's exceptions, once: positions within a chunk become (row, column)
  // relative to the CTA's tile with 32-bit arithmetic when 128 K fits it,
  // counted per stage, then binned by stage so that each stage's are found
  // without a search and patched by the thread that expanded their segment.
  const uint64_t f_base = uint64_t(n0) * K, f_span = uint64_t(kBM) * K;
  const uint32_t k_beg = s_begin * kBK, k_end = s_end * kBK;
  // The chunks' lists follow one another in the container, so the row
  // block's exceptions are the one range [exc_off[c_lo], exc_off[c_hi + 1]);
  // its entries are taken by all threads at once, each finding its chunk by
  // a search in a shared copy of the offsets (up to kGatherChunks chunks;
  // beyond that, chunk after chunk).
  const uint32_t nch = uint32_t(c_hi - c_lo + 1);
  auto gather_one = [&](uint64_t c, uint64_t e, uint32_t pos) {
    const uint64_t cnt = n - c * kChunk < kChunk ? n - c * kChunk : kChunk;
    if (pos >= cnt) {
      report(p.status, WC_ERR_CORRUPT);
      return;
    }
    const uint64_t f = c * kChunk + pos;
    if (f < f_base || f - f_base >= f_span) return;
    const uint64_t lf = f - f_base;
    uint32_t row, col;
    if (f_span <= 0xFFFFFFFFull) {
      row = uint32_t(lf) / K;
      col = uint32_t(lf) - row * K;
    } else {
      row = uint32_t(lf / K);
      col = uint32_t(lf - uint64_t(row) * K);
    }
    if (col < k_beg || col >= k_end) return;
    const uint32_t slot = atomicAdd(exc_n, 1u);
    if (slot < kExcCap) {
      exc_raw[slot] = make_uint2(col - k_beg, row | (uint32_t(exc_val[e]) << 16));
      if (binned) atomicAdd(&bin[(col - k_beg) / kBK], 1u);
    }
  };
  if (nch <= kGatherChunks) {
    for (uint32_t j = tid; j <= nch; j += kThreads) g_off[j] = exc_off[c_lo + j];
    __syncthreads();
    bool bad = false;
    for (uint32_t j = tid; j < nch; j += kThreads) bad |= g_off[j] > g_off[j + 1] || g_off[j + 1] > ne;
    if (__syncthreads_or(bad)) {
      if (tid == 0) report(p.status, WC_ERR_CORRUPT);
    } else {
      const uint64_t e_beg = g_off[0], e_end = g_off[nch];
      constexpr uint32_t kG = 4;  // positions loaded together
      for (uint64_t e = e_beg + tid; e < e_end; e += kThreads * kG) {
        uint32_t pos[kG];
#pragma unroll
        for (uint32_t u = 0; u < kG; u++) {
          const uint64_t eu = e + uint64_t(u) * kThreads;
          pos[u] = eu < e_end ? exc_pos[eu] : 0u;
        }
#pragma unroll
        for (uint32_t u = 0; u < kG; u++) {
          const uint64_t eu = e + uint64_t(u) * kThreads;
          if (eu >= e_end) break;
          uint32_t lo = 0, hi = nch - 1;  // the last chunk j with g_off[j] <= eu
          while (lo < hi) {
            const uint32_t mid = (lo + hi + 1) >> 1;
            if (g_off[mid] <= eu) lo = mid; else hi = mid - 1;
          }
          gather_one(c_lo + lo, eu, pos[u]);
        }
      }
    }
  } else {
    for (uint64_t c = c_lo; c <= c_hi; c++) {
      const uint64_t e0 = exc_off[c], e1 = exc_off[c + 1];
      if (e0 > e1 || e1 > ne) {
        if (tid == 0) report(p.status, WC_ERR_CORRUPT);
        continue;
      }
      for (uint64_t e = e0 + tid; e < e1; e += kThreads) gather_one(c, e, exc_pos[e]);
    }
  }
  __syncthreads();
  const uint32_t n_exc = *exc_n;
  mode = n_exc > kExcCap || !binned ? 2 : 0;
  if (mode == 0) {
    // counts -> starts (one warp), then scatter by stage
    if (warp == 0) {
      uint32_t run = 0;
      for (uint32_t b0 = 0; b0 <= nst; b0 += 32) {
        const uint32_t b = b0 + lane;
        const uint32_t v = b < nst ? bin[b] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        if (b <= nst) bin[b] = run + incl - v;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();
    for (uint32_t i = tid; i <= nst; i += kThreads) cur[i] = bin[i];
    __syncthreads();
    for (uint32_t i = tid; i < n_exc; i += kThreads) {
      const uint2 ex = exc_raw[i];  // column in the CTA's range -> in its stage
      exc_bin[atomicAdd(&cur[ex.x / kBK], 1u)] = make_uint2(ex.x % kBK, ex.y);
    }
    __syncthreads();
  }
  }

  // The pipeline.  Expanding threads, stage s: wait for slot s % kDepth's
  // loads and for A slot s % 2 to be free (the MMAs of stage s - 2), expand
  // into it, arrive on its a_full; then load stage s + kDepth - 1 into the
  // slot stage s - 1 used, once that stage's MMAs are done.  The MMA thread,
  // stage s: wait for a_full, issue the four MMAs, commit them to a_free and
  // slot_free.  No block-wide barrier inside the loop.
  const volatile int *vflag = flag;
  uint32_t issued = 0;  // MMA thread: stages whose MMAs were issued
  if (expander) {
    // this thread's two segments: offsets of their index and low bytes in a
    // ring slot and of their two 16-byte rows in an A slot
    uint32_t o_idx[2], o_lo[2], o_a[2];
#pragma unroll
    for (int q = 0; q < 2; q++) {
      const uint32_t i = uint32_t(tid) + kExpThreads * q, row = ((i >> 5) << 3) | (i & 7), seg = (i >> 3) & 3;
      o_idx[q] = idx_gran(row, seg >> 1) + 8 * (seg & 1);
      o_lo[q] = kIdxBytes + lo_gran(row, seg);
      o_a[q] = op_offset(row, 16 * seg, kASlice);  // + 128: the segment's second 8 values
    }
    // mode 1: bounds of the current stage and this thread's first entry of it
    uint32_t pb0 = 0, pb1 = 0, pe = 0;
    if (mode == 1) {
      pb0 = plan_start[0];
      pb1 = plan_start[1];
      pe = pb0 + uint32_t(tid) < ne ? plan_ent[pb0 + tid] : 0u;
    }
    for (uint32_t s = 0; s < nst; s++) {
      const uint32_t as = s % kASlots;
      uint8_t *A = a_op + as * kAStage;
      const uint8_t *slot = ring + (s % kDepth) * sb;
      // the stage's loads have landed; A slot s % 2 is free once the MMAs of
      // stage s - 2 are done
      const bool okw = mbar_wait_or_flag(&full[s % kDepth], (s / kDepth) & 1u, vflag) &&
                       (s < kASlots || mbar_wait_or_flag(&a_free[as], ((s / kASlots) & 1u) ^ 1u, vflag));
      const uint32_t k0 = (s_begin + s) * kBK;
      uint32_t eb0 = 0, eb1 = 0, first_e = 0;  // the stage's exceptions (modes 0, 1)
      if (mode == 0) {
        eb0 = bin[s];
        eb1 = bin[s + 1];
      } else if (mode == 1) {
        // this stage's bounds and entry, read during the previous one; the
        // next stage's now (the entry speculatively, within the plan)
        eb0 = pb0;
        eb1 = pb1;
        first_e = pe;
        pb0 = pb1;
        pb1 = s + 2 <= nst ? plan_start[s + 2] : pb1;
        pe = eb1 + uint32_t(tid) < ne ? plan_ent[eb1 + tid] : 0u;
      }
      if (okw) {
        // A: 512 segments of 16 values, two per thread: segment i is row
        // 8 (i / 32) + i % 8, values 16 ((i / 8) % 4) .., expanded from the
        // ring slot into the operand slot
#pragma unroll
        for (int q = 0; q < 2; q++) {
          const uint2 iw = *reinterpret_cast<const uint2 *>(slot + o_idx[q]);
          const uint4 lw = *reinterpret_cast<const uint4 *>(slot + o_lo[q]);
          const uint2 e0 = wc12::expand4(iw.x, book, lw.x), e1 = wc12::expand4(iw.x >> 16, book, lw.y);
          const uint2 e2 = wc12::expand4(iw.y, book, lw.z), e3 = wc12::expand4(iw.y >> 16, book, lw.w);
          *reinterpret_cast<uint4 *>(A + o_a[q]) = make_uint4(e0.x, e0.y, e1.x, e1.y);
          *reinterpret_cast<uint4 *>(A + o_a[q] + 128) = make_uint4(e2.x, e2.y, e3.x, e3.y);
        }
      }
      // The expanders meet (named barrier 1): every segment of the stage is
      // written, and all decide together whether to go on.
      if (!expanders_all(okw)) {
        if (!*vflag) report(p.status, WC_ERR_TIMEOUT);
        *flag = 1;
        break;
      }
      // the exceptions that fall in this tile get their high bytes, one
      // thread an exception
      if (mode == 0) {
        for (uint32_t i = eb0 + uint32_t(tid); i < eb1; i += kExpThreads) {
          const uint2 ex = exc_bin[i];
          A[op_offset(ex.y & 0xFFFFu, ex.x, kASlice) + 1] = uint8_t(ex.y >> 16);
        }
      } else if (mode == 1) {
        if (eb0 > eb1 || eb1 > ne) {
          if (tid == 0) report(p.status, WC_ERR_CORRUPT);
        } else {
          for (uint32_t i = eb0 + uint32_t(tid); i < eb1; i += kExpThreads) {
            const uint32_t e = i == eb0 + uint32_t(tid) ? first_e : plan_ent[i];
            A[op_offset((e >> 6) & 127u, e & 63u, kASlice) + 1] = uint8_t(e >> 16);
          }
        }
      } else if (mode == 2) {
        for (uint64_t c = c_lo; c <= c_hi; c++) {
          const uint64_t e0 = exc_off[c], e1 = exc_off[c + 1];
          if (e0 > e1 || e1 > ne) continue;  // reported by the gathering pass
          const uint64_t cnt = n - c * kChunk < kChunk ? n - c * kChunk : kChunk;
          for (uint64_t e = e0 + tid; e < e1; e += kExpThreads) {
            const uint32_t pos = exc_pos[e];
            if (pos >= cnt) continue;
            const uint64_t f = c * kChunk + pos;
            const uint64_t row = f / K, col = f % K;
            if (row < n0 || row >= n0 + kBM || col < k0 || col >= k0 + kBK) continue;
            A[op_offset(uint32_t(row - n0), uint32_t(col - k0), kASlice) + 1] = exc_val[e];
          }
        }
      }
      fence_proxy_async();  // generic-proxy writes -> visible to the tensor cores
      mbar_arrive(&a_full[as]);
    }
  } else if (warp == kMmaWarp && lane == 0) {
    const uint32_t idesc = instr_desc(p.n_mma);
    for (uint32_t s = 0; s < nst; s++) {
      const uint32_t as = s % kASlots;
      if (!mbar_wait_or_flag(&a_full[as], (s / kASlots) & 1u, vflag)) {
        if (!*vflag) report(p.status, WC_ERR_TIMEOUT);
        *flag = 1;
        break;
      }
      fence_after_sync();
      const uint32_t a0 = smem_u32(a_op + as * kAStage), b0 = ring_s + (s % kDepth) * sb + kIdxBytes + kLoBytes;
#pragma unroll
      for (uint32_t sl = 0; sl < 4; sl++)
        mma_bf16(tmem, operand_desc(a0 + sl * kASlice, 128, 256, 0), operand_desc(b0 + 32 * sl, 16, 1024, 2),
                 idesc, (s > 0 || sl > 0) ? 1u : 0u);
      mma_commit(&a_free[as]);
      mma_commit(&slot_free[s % kDepth]);
      issued = s + 1;
    }
  } else if (loader) {
    // stage j reuses the slot of stage j - kDepth once its MMAs are done
    for (; loaded < nst; loaded++) {
      const uint32_t prev = loaded - kDepth;
      if (!mbar_wait_or_flag(&slot_free[prev % kDepth], (prev / kDepth) & 1u, vflag)) {
        if (!*vflag) report(p.status, WC_ERR_TIMEOUT);
        *flag = 1;
        break;
      }
      load_stage(loaded);
    }
    // no load may still be in flight when the CTA ends: wait (bounded, also
    // after a failure) for the last stage issued into each slot
    for (uint32_t j = loaded > kDepth ? loaded - kDepth : 0; j < loaded; j++)
      if (!mbar_wait(&full[j % kDepth], (j / kDepth) & 1u)) report(p.status, WC_ERR_TIMEOUT);
  }

  // The MMA thread waits for the last stage it issued (the commit covers all
  // earlier MMAs), without giving up on a flag: tensor memory is read and
  // freed only after its MMAs are done.
  bool done = true;
  if (warp == kMmaWarp && lane == 0 && issued > 0) {
    const uint32_t last = issued - 1;
    done = mbar_wait(&slot_free[last % kDepth], (last / kDepth) & 1u);
  }
  if (!expander) __syncwarp();
  // every thread takes the same branch below: the tensor-memory loads are
  // warp-collective (.sync.aligned)
  done = __syncthreads_and(done) != 0;
  if (!done && tid == kExpThreads) report(p.status, WC_ERR_TIMEOUT);
  fence_after_sync();
  if (done && !*flag && expander) {
    // warp w reads TMEM lanes 32 (w % 4) .. (its rows); warps 0-3 take the
    // even 8-column groups, warps 4-7 the odd ones
    const uint32_t lane_base = 32 * (warp & 3);
    const uint32_t row = n0 + lane_base + lane;
    for (uint32_t c0 = 8 * (warp >> 2); c0 < p.n_mma; c0 += 16) {
      uint32_t v[8];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
          : "r"(tmem + (lane_base << 16) + c0));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const uint32_t t = c0 + i;
        if (t < p.M) {
          float *dst = p.y + uint64_t(t) * N + row;
          if (p.splits > 1) atomicAdd(dst, __uint_as_float(v[i]));
          else *dst = __uint_as_float(v[i]);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols) : "memory");
  }
}

// ---------------------------------------------------------------------------
__global__ void k12_zero(float *y, uint64_t count) {
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += uint64_t(gridDim.x) * blockDim.x)
    y[i] = 0.0f;
}

struct DevInfo {
  int sms = 0;
  bool attr = false;
  int smem_per_sm = 0;     // shared memory of one SM
  int smem_reserved = 0;   // per CTA, taken by the system
  int regs[4] = {};  // registers a thread of each compiled shape (kShapes)
  unsigned long long ctx = 0;  // the context the attributes were set in
};

// The compiled pipeline shapes {ring depth, A slots}, deepest first.
struct Shape {
  uint32_t depth, aslots;
};
constexpr Shape kShapes[4] = {{4, 2}, {3, 2}, {2, 2}, {2, 1}};

using LinearKernel = void (*)(Params);
LinearKernel kernel_for(uint32_t shape) {
  switch (shape) {
    case 1: return k12_linear<3, 2>;
    case 2: return k12_linear<2, 2>;
    case 3: return k12_linear<2, 1>;
    default: return k12_linear<4, 2>;
  }
}

// The shape of a launch: the first of kShapes (a 4-, 3- or 2-slot ring with
// two A slots, then a 2-slot ring with one A slot, whose expansion of a stage
// waits for the MMAs of the one before) that lets two CTAs share an SM —
// two pipelines an SM, and every SM busy — else the deepest, one CTA an SM.
uint32_t pick_shape(const DevInfo &d, uint32_t n_mma, bool plan) {
  for (uint32_t i = 0; i < 4; i++)
    if (2 * (smem_bytes(n_mma, kShapes[i].depth, kShapes[i].aslots, plan) + uint32_t(d.smem_reserved)) <=
        uint32_t(d.smem_per_sm))
      return i;
  return 0;
}

// Dynamic shared memory for a launch with n_mma token columns and pipeline
// shape `shape`: at least what the stages need, padded so that the CTAs that
// fit on one SM hold at most the SM's 512 tensor-memory columns between them
// (otherwise a CTA's tcgen05.alloc would wait for another CTA to finish).
uint32_t launch_smem(const DevInfo &d, uint32_t n_mma, uint32_t shape, bool plan) {
  uint32_t cols = 32;
  while (cols < n_mma) cols <<= 1;
  const uint32_t max_ctas = 512 / cols;
  uint32_t need = smem_bytes(n_mma, kShapes[shape].depth, kShapes[shape].aslots, plan);
  const uint32_t per_sm = uint32_t(d.smem_per_sm), rsv = uint32_t(d.smem_reserved);
  // CTAs per SM = floor(per_sm / (smem + rsv)); make it <= max_ctas
  const uint32_t floor_smem = per_sm / (max_ctas + 1) + 1;
  if (floor_smem > rsv && need + rsv < floor_smem) need = floor_smem - rsv;
  return need;
}

// cuTensorMapEncodeTiled, from the driver (once)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A 2-D map over rows of `inner` elements, `row_bytes` apart, loaded in
// boxes of box_rows x box_inner.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw,
              CUtensorMapL2promotion l2) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, l2,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

DevInfo dev_info() {
  static std::mutex mu;
  static DevInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DevInfo{};
  std::lock_guard<std::mutex> lock(mu);
  DevInfo &d = cache[dev];
  // once per device, and again in a context created afresh (after a
  // cudaDeviceReset the kernels' shared-memory attributes must be set again)
  const unsigned long long ctx = wc::current_context_id();
  if (d.sms == 0 || (ctx != 0 && d.ctx != ctx)) {
    d = DevInfo{};
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DevInfo{};
    int per_sm = 0, rsv = 0;
    if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
      return DevInfo{};
    d.smem_per_sm = per_sm;
    d.smem_reserved = rsv;
    d.attr = true;
    for (uint32_t i = 0; i < 4; i++) {
      uint32_t most = 0;  // the largest launch of this shape (without a plan: the exception list)
      for (uint32_t m = 16; m <= kMaxTokens; m += 16) {
        const uint32_t b = launch_smem(d, m, i, false);
        most = b > most ? b : most;
      }
      d.attr = d.attr && cudaFuncSetAttribute(kernel_for(i), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              int(most)) == cudaSuccess;
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, kernel_for(i)) != cudaSuccess) return DevInfo{};
      d.regs[i] = fa.numRegs;
    }
    d.sms = sms;
    d.ctx = wc::current_context_id();  // the set-up made the device's context current
  }
  return d;
}

}  // namespace wc12l

namespace wc12l {

int32_t linear(const void *d_w, uint64_t w_bytes, const void *d_plan, uint64_t plan_bytes, uint32_t N,
               uint32_t K, const void *d_x, uint32_t M, float *d_y, int32_t *d_status, void *stream) {
  auto aligned = [](const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; };
  if (d_w == nullptr || d_x == nullptr || d_y == nullptr || d_status == nullptr) return WC_ERR_INVALID_ARG;
  if (!aligned(d_w, 16) || !aligned(d_x, 16) || !aligned(d_y, 4) || !aligned(d_status, 4))
    return WC_ERR_INVALID_ARG;
  if (N == 0 || K == 0 || N % wc12l::kBM != 0 || K % wc12l::kBK != 0 || M == 0)
    return WC_ERR_INVALID_ARG;
  if (w_bytes < 96) return WC_ERR_INVALID_ARG;  // shorter than any container's header
  // the index and low planes of an N x K container must lie inside the
  // buffer (their offsets depend on N K only; the kernels check the header)
  const uint64_t n = uint64_t(N) * K;
  const wc12::Lay L = wc12::lay(n, 0);
  if (w_bytes < L.off_lo + n) return WC_ERR_INVALID_ARG;
  if (d_plan != nullptr &&
      (!aligned(d_plan, 16) || plan_bytes < wc12p::plan_lay(N, K, 0).off_ent))  // header and starts
    return WC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  wc12l::Params p;
  p.w = static_cast<const uint8_t *>(d_w);
  p.w_bytes = w_bytes;
  p.plan = static_cast<const uint8_t *>(d_plan);
  p.plan_bytes = plan_bytes;
  p.N = N;
  p.K = K;
  p.status = d_status;
  const wc12l::DevInfo di = wc12l::dev_info();
  if (di.sms <= 0 || !di.attr) return WC_ERR_CUDA;
  const uint32_t blocks = N / wc12l::kBM, stages = K / wc12l::kBK;
  if (blocks == 0) return WC_ERR_INVALID_ARG;
  if (!wc12l::make_map(&p.tm_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.w + L.off_idx, K / 2, N, K / 2, 32,
                       wc12l::kBM, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !wc12l::make_map(&p.tm_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.w + L.off_lo, K, N, K, 64, wc12l::kBM,
                       CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return WC_ERR_CUDA;
  // tokens in slices of at most kMaxTokens (the MMA's N); each slice's rows
  // of X and Y are contiguous
  for (uint32_t t0 = 0; t0 < M; t0 += wc12l::kMaxTokens) {
    const uint32_t m = M - t0 < wc12l::kMaxTokens ? M - t0 : wc12l::kMaxTokens;
    p.x = static_cast<const uint16_t *>(d_x) + uint64_t(t0) * K;
    p.y = d_y + uint64_t(t0) * N;
    p.M = m;
    p.n_mma = (m + 15) / 16 * 16;
    if (!wc12l::make_map(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, K, m, uint64_t(K) * 2, wc12l::kBK, p.n_mma,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
      return WC_ERR_CUDA;
    // split K so that the grid is one wave of the CTAs an SM holds, with at
    // least 4 stages a CTA when K allows (the load ring runs up to 4 ahead)
    const uint32_t shape = wc12l::pick_shape(di, p.n_mma, d_plan != nullptr);
    const uint32_t smem = wc12l::launch_smem(di, p.n_mma, shape, d_plan != nullptr);
    uint32_t cols = 32;
    while (cols < p.n_mma) cols <<= 1;
    // CTAs an SM holds: shared memory, registers (whole warps of 8-register
    // granules), threads, and the two the kernel is compiled for
    uint32_t per_sm = uint32_t(di.smem_per_sm) / (smem + uint32_t(di.smem_reserved));
    const uint32_t warp_regs = (uint32_t(di.regs[shape]) + 7) / 8 * 8 * 32;
    const uint32_t by_regs = 65536 / (warp_regs * (wc12l::kThreads / 32));
    if (per_sm > by_regs) per_sm = by_regs;
    if (per_sm > 2048 / wc12l::kThreads) per_sm = 2048 / wc12l::kThreads;
    if (per_sm > 2) per_sm = 2;
    if (per_sm > 512 / cols) per_sm = 512 / cols;
    if (per_sm < 1) per_sm = 1;
    uint32_t splits = uint32_t(di.sms) * per_sm / blocks;
    const uint32_t most = stages / 4 > 0 ? stages / 4 : 1;
    if (splits > most) splits = most;
    if (splits < 1) splits = 1;
    p.per_split = (stages + splits - 1) / splits;
    p.splits = (stages + p.per_split - 1) / p.per_split;
    if (p.splits > 1) wc12l::k12_zero<<<unsigned(2 * di.sms), 256, 0, s>>>(p.y, uint64_t(m) * N);
    dim3 grid(blocks, p.splits);
    wc12l::kernel_for(shape)<<<grid, wc12l::kThreads, smem, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return WC_ERR_CUDA;
  }
  return WC_OK;
}

}  // namespace wc12l

extern "C" int32_t wc12_linear(const void *d_w, uint64_t w_bytes, uint32_t N, uint32_t K,
                               const void *d_x, uint32_t M, float *d_y, int32_t *d_status,
                               void *stream) {
  return wc12l::linear(d_w, w_bytes, nullptr, 0, N, K, d_x, M, d_y, d_status, stream);
}

extern "C" int32_t wc12_linear_planned(const void *d_w, uint64_t w_bytes, const void *d_plan,
                                       uint64_t plan_bytes, uint32_t N, uint32_t K, const void *d_x,
                                       uint32_t M, float *d_y, int32_t *d_status, void *stream) {
  if (d_plan == nullptr) return WC_ERR_INVALID_ARG;
  return wc12l::linear(d_w, w_bytes, d_plan, plan_bytes, N, K, d_x, M, d_y, d_status, stream);
}

