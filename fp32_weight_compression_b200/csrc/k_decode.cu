// k_decode.cu -- decoder: rANS decode of the exponent chunks fused with the
// re-merge of the planes into the original bits ("PTWM" How it works 1-2 run
// backwards; "SMEF" pass3_streams.py merge_streams).
//
// Persistent grid of 8-warp blocks.  Work is split into groups of 16
// consecutive chunks of one tensor; a block takes the next group from the
// launch's counter whenever it has finished one (the blocks an SM holds do
// not progress at one rate -- measured, the slowest block of an SM took
// ~30 % longer per group than the fastest -- so a fixed share each would
// leave the fast blocks idle while the slow ones finish).
// The block stages its tensor's 4096-slot decoding table in
// shared memory (entry = symbol | (slot - cum) << 8 | f << 20) and each warp
// decodes two chunks.  When both are full 65,536-symbol coded chunks the warp
// runs them in lock-step, so every lane carries two independent state chains;
// otherwise it decodes them one after the other.  One decoding step:
//   slot = x & 4095; e = tab[slot]; x = f (x >> 12) + (slot - cum);
//   if x < 2^16: x = x << 16 | next word
// The lanes that need a word at a step take consecutive words in lane order
// (__ballot_sync / __popc prefix), from a per-chunk 1024-word shared-memory
// ring that cp.async keeps filled with 16-byte loads of the chunk's word
// stream.  Every 8 steps a chunk has 256 new coded bytes; they are transposed
// through shared memory so that each lane holds 8 consecutive ones, merged
// with the matching raw-plane bytes, and written with one 16-byte store (bf16,
// fp16), two (fp32) or one 8-byte store (fp8).
//
// Everything read from the container is checked before use (header fields
// against the layout implied by n, the table sum, each chunk's offset pair and
// length); a decoded chunk must end with every lane at 2^16 and every word
// consumed.  Failures store a wc_status code in *status and skip the chunk.
// No loop waits on another block; each wait is on this warp's own copies.
#include <atomic>
#include <mutex>

#include "wc_block.cuh"
#include "wc_format.cuh"
#include "wc_planes.cuh"

namespace wc {

constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kDecGroup = kDecWarps * 2;  // most chunks per block group
constexpr uint32_t kRing = 1024;                // words per chunk ring
constexpr uint32_t kUnit = 256;                 // words per cp.async round (32 lanes x 16 B)
constexpr uint32_t kHalf = 256;                 // values per half-group (8 steps)

struct DecSmem {
  uint32_t tab[kProbScale];                          // 16 KiB
  __align__(16) uint8_t tbuf[kDecWarps][2][kHalf];   // 4 KiB
  uint32_t gpre[kMaxItems + 1];
  uint64_t red[kDecThreads / 32 + 1];
  int cur_item;
  uint32_t next_grp;
  int tab_ok;
  int single_sym;
  // Word rings, kRing u16 per chunk, each on a 2 KiB boundary of the shared
  // window (the slack lets ring_ptr align them at run time); freq/cum while a
  // table is built.
  __align__(16) uint8_t ring_raw[kDecWarps * 2 * kRing * 2 + 2048];
};

// The block's dynamic shared memory (a DecSmem).  Functions below reach it
// through this symbol, not through pointer arguments, so that every access
// compiles to a shared-memory instruction.
extern __shared__ __align__(16) uint8_t dyn_smem[];
__device__ __forceinline__ DecSmem &smem() { return *reinterpret_cast<DecSmem *>(dyn_smem); }

// Ring of chunk slot c of warp w.
__device__ __forceinline__ uint16_t *ring_ptr(int w, int c) {
  uint8_t *r = smem().ring_raw;
  const uint32_t a = uint32_t(__cvta_generic_to_shared(r));
  const uint32_t pad = ((a + 2047u) & ~2047u) - a;
  return reinterpret_cast<uint16_t *>(r + pad + (w * 2 + c) * kRing * 2);
}

__device__ __forceinline__ void report(int32_t *status, int32_t code) {
  atomicCAS(status, 0, code);
}

struct ItemView {
  bool ok;
  int32_t err;
  int dtype;
  uint64_t n;
  Layout L;
  uint64_t first, cnt;  // chunk range
};

// Header checks that need no table or chunk data.
__device__ __noinline__ ItemView view_item(const DecItem &it) {
  ItemView v;
  v.ok = false;
  v.err = WC_ERR_CORRUPT;
  v.first = v.cnt = 0;
  v.n = 0;
  v.dtype = 0;
  if (it.cont_bytes < kChunkOffOffset + 16) return v;
  const uint32_t *h32 = reinterpret_cast<const uint32_t *>(it.cont);
  const uint64_t *h64 = reinterpret_cast<const uint64_t *>(it.cont);
  const uint32_t w1 = h32[1];
  const int dtype = int((w1 >> 16) & 0xFF);
  if (h32[0] != 0x315A4357u || (w1 & 0xFFFF) != kVersion || (w1 >> 24) != kLanes) return v;
  if (dtype != WC_BF16 && dtype != WC_FP32 && dtype != WC_FP16 && !is_fp8(dtype)) return v;
  const uint64_t n = h64[1];
  if (n > (uint64_t(1) << 44)) return v;
  if (h32[4] != kChunk || h32[6] != kProbBits || h32[7] != 0) return v;
  const Layout L = make_layout(n, dtype);
  if (h32[5] != uint32_t(L.nc) || h64[4] != L.off_raw || h64[5] != L.off_exp) return v;
  const uint64_t exp_bytes = h64[6], total = h64[7];
  if (it.cont_bytes < L.off_exp || total != L.off_exp + exp_bytes || total > it.cont_bytes) return v;
  v.dtype = dtype;
  v.n = n;
  v.L = L;
  if (it.chunk_count == ~uint64_t(0)) {
    v.first = 0;
    v.cnt = L.nc;
  } else {
    if (it.chunk_first >= L.nc) { v.err = WC_ERR_INVALID_ARG; return v; }
    v.first = it.chunk_first;
    v.cnt = min(it.chunk_count, L.nc - it.chunk_first);
  }
  const uint64_t elem = dtype_bytes(dtype);
  const uint64_t vals = v.cnt == 0 ? 0
                        : (v.first + v.cnt == L.nc ? n - v.first * kChunk : v.cnt * kChunk);
  if (vals * elem > it.out_cap || (vals > 0 && it.out == nullptr)) { v.err = WC_ERR_CAPACITY; return v; }
  v.ok = true;
  v.err = WC_OK;
  return v;
}

// A chunk's offset-table entry, checked.
struct ChunkView {
  bool ok, raw;
  uint32_t nsym, len;
  const uint8_t *pay;  // payload in the exponent section
  uint8_t *out;        // output slot of the chunk's first value
};

template <int DT>
__device__ __forceinline__ ChunkView view_chunk(const DecItem &it, const ItemView &v, uint64_t k) {
  ChunkView c;
  const Layout &L = v.L;
  const uint8_t *cont = it.cont;
  c.nsym = chunk_nsym(v.n, k);
  const uint64_t *choff = reinterpret_cast<const uint64_t *>(cont + L.off_chunk_off);
  const uint32_t *chlen = reinterpret_cast<const uint32_t *>(cont + L.off_chunk_len);
  const uint64_t exp_bytes = reinterpret_cast<const uint64_t *>(cont)[6];
  const uint64_t o0 = choff[k], o1 = choff[k + 1];
  c.len = chlen[k];
  c.raw = c.len == c.nsym;
  const bool coded = c.len >= kStateBytes && c.len < c.nsym && (c.len & 1u) == 0;
  c.ok = (c.raw || coded) && o0 <= o1 && o1 - o0 == round16(c.len) && o1 <= exp_bytes &&
         (k != 0 || o0 == 0) && (k + 1 != L.nc || o1 == exp_bytes);
  c.pay = cont + L.off_exp + o0;
  constexpr uint32_t elem = dtype_bytes(DT);
  c.out = it.out + (k - v.first) * kChunk * elem;
  return c;
}

// ---------------------------------------------------------------------------
// Raw-plane bytes of 8 consecutive values and the merge.
template <int DT>
struct Raw8 {
  uint2 a;        // bf16 / fp16: the 8 raw bytes; fp8: a.x = 8 packed nibbles;
                  // fp32: mantissa bytes 0..7
  uint2 b, c;     // fp32: mantissa bytes 8..23
  uint32_t s;     // fp32: 8 sign bits
};

template <int DT>
__device__ __forceinline__ void load_raw8(const uint8_t *cont, const Layout &L, uint64_t vg, Raw8<DT> &r) {
  if (is_fp8(DT)) {
    r.a.x = __ldg(reinterpret_cast<const uint32_t *>(cont + L.off_raw + vg / 2));
  } else if (DT != WC_FP32) {
    r.a = __ldg(reinterpret_cast<const uint2 *>(cont + L.off_raw + vg));
  } else {
    r.s = __ldg(cont + L.off_raw + vg / 8);
    const uint2 *m = reinterpret_cast<const uint2 *>(cont + L.off_mant + 3 * vg);
    r.a = __ldg(m);
    r.b = __ldg(m + 1);
    r.c = __ldg(m + 2);
  }
}

// fp32 value j of 4 from 3 mantissa words: u = s << 31 | e << 23 | m
__device__ __forceinline__ uint4 merge4_fp32(uint32_t e4, uint32_t w0, uint32_t w1, uint32_t w2,
                                             uint32_t s4) {
  const uint32_t m0 = w0 & 0x7FFFFFu;
  const uint32_t m1 = __funnelshift_r(w0, w1, 24) & 0x7FFFFFu;
  const uint32_t m2 = __funnelshift_r(w1, w2, 16) & 0x7FFFFFu;
  const uint32_t m3 = (w2 >> 8) & 0x7FFFFFu;
  uint4 o;
  o.x = ((s4 & 1u) << 31) | ((e4 & 0xFFu) << 23) | m0;
  o.y = ((s4 & 2u) << 30) | (((e4 >> 8) & 0xFFu) << 23) | m1;
  o.z = ((s4 & 4u) << 29) | (((e4 >> 16) & 0xFFu) << 23) | m2;
  o.w = ((s4 & 8u) << 28) | ((e4 >> 24) << 23) | m3;
  return o;
}

// 8 values (coded bytes e8 = 8 bytes) -> output at dst (16-byte aligned);
// 2-byte values merge byte-parallel (merge4, wc_planes.cuh).
template <int DT>
__device__ __forceinline__ void merge_store8(uint2 e8, const Raw8<DT> &r, uint8_t *dst) {
  if (is_fp8(DT)) {
    st_cs_v2(dst, fp8_merge8<DT>(e8, r.a.x));  // 8 one-byte values
  } else if (DT != WC_FP32) {
    const uint2 p = merge4<DT>(e8.x, r.a.x);
    const uint2 q = merge4<DT>(e8.y, r.a.y);
    st_cs_v4(dst, make_uint4(p.x, p.y, q.x, q.y));
  } else {
    // mantissa words: a.x a.y b.x | b.y c.x c.y
    st_cs_v4(dst, merge4_fp32(e8.x, r.a.x, r.a.y, r.b.x, r.s));
    st_cs_v4(dst + 16, merge4_fp32(e8.y, r.b.y, r.c.x, r.c.y, r.s >> 4));
  }
}

// One value, for ragged tails (scalar; no register arrays).
template <int DT>
__device__ __forceinline__ void merge_store1(uint32_t e, const uint8_t *cont, const Layout &L, uint64_t vg,
                                             uint8_t *dst) {
  if (is_fp8(DT)) {
    dst[0] = uint8_t(fp8_merge<DT>(e, (cont[L.off_raw + vg / 2] >> (4 * (vg & 1))) & 0xFu));
  } else if (DT != WC_FP32) {
    reinterpret_cast<uint16_t *>(dst)[0] = uint16_t(merge16<DT>(e, cont[L.off_raw + vg]));
  } else {
    const uint32_t s = (cont[L.off_raw + vg / 8] >> (vg & 7)) & 1u;
    const uint8_t *m = cont + L.off_mant + 3 * vg;
    const uint32_t mant = (uint32_t(m[0]) | uint32_t(m[1]) << 8 | uint32_t(m[2]) << 16) & 0x7FFFFFu;
    reinterpret_cast<uint32_t *>(dst)[0] = (s << 31) | (e << 23) | mant;
  }
}

// ---------------------------------------------------------------------------
// The word ring of one chunk.
struct Ring {
  uint32_t rs;         // shared address of the ring
  const uint8_t *src;  // first word
  uint32_t avail;      // readable words (payload rounded to 16 bytes)
  uint32_t req;        // words requested so far (multiple of kUnit)
  uint32_t f1, f2;     // requested frontier after the call before last / before that
  uint32_t landed;     // words known to be in shared memory (after a wait)

  __device__ __forceinline__ void issue(int lane) {
    const uint32_t j0 = req + 8 * lane;
    const uint32_t dst = rs + ((j0 & (kRing - 1)) << 1);
    if (j0 < avail) cp_async16_s(dst, src + 2 * j0, 16);
    else cp_async16_s(dst, src, 0);  // zero fill, reads nothing
    req += kUnit;
  }
  // Called once per half-group, followed by one commit.  Issues the next unit
  // if it fits without overwriting unread words (a half-group consumes at
  // most one unit, so the requested frontier stays >= cons + 513 words).
  // Returns how many of the most recent commit groups may still be in flight
  // while the words [cons, cons + 256) are already in shared memory: 3 if
  // they were requested three calls ago or earlier, ..., 0 if only now.
  __device__ __forceinline__ int top_up(uint32_t cons, int lane) {
    const uint32_t f0 = top(cons, lane);
    const int d = depth(min(cons + kHalf, avail), f0);
    shift(f0);
    return d;
  }
  // The same in parts, for a caller that skips the wait while the words it
  // needs are known to have landed: top() issues and returns the frontier
  // before this call; depth(); frontier(d) is what a wait at depth d
  // guarantees; shift() moves the history on.
  __device__ __forceinline__ uint32_t top(uint32_t cons, int lane) {
    const uint32_t f0 = req;  // frontier after the previous call
    if (req < avail && req + kUnit <= (cons & ~(kUnit - 1)) + kRing) issue(lane);
    return f0;
  }
  __device__ __forceinline__ int depth(uint32_t need, uint32_t f0) const {
    return f2 >= need ? 3 : (f1 >= need ? 2 : (f0 >= need ? 1 : 0));
  }
  __device__ __forceinline__ uint32_t frontier(int d, uint32_t f0) const {
    return d >= 3 ? f2 : (d == 2 ? f1 : (d == 1 ? f0 : req));
  }
  __device__ __forceinline__ void shift(uint32_t f0) {
    f2 = f1;
    f1 = f0;
  }
};

__device__ __forceinline__ void cp_async_wait_depth(int d) {
  if (d >= 3) cp_async_wait<3>();
  else if (d == 2) cp_async_wait<2>();
  else if (d == 1) cp_async_wait<1>();
  else cp_async_wait<0>();
}

// One decoding step of one lane.
__device__ __forceinline__ void dstep(uint32_t &x, uint32_t &cons, const uint32_t *tab,
                                      const uint16_t *ring, uint8_t *tbp, uint32_t lt) {
  const uint32_t e = tab[x & (kProbScale - 1)];
  x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
  const bool rn = x < kStateLow;
  const uint32_t m = __ballot_sync(0xffffffffu, rn);
  const uint32_t w = ring[(cons + __popc(m & lt)) & (kRing - 1)];
  const uint32_t xr = __byte_perm(x, w, 0x1054);  // x << 16 | w
  x = rn ? xr : x;
  cons += __popc(m);
  *tbp = uint8_t(e);
}

// Where a chunk's raw planes start, per dtype (value 0 of the chunk).
struct RawPtrs {
  const uint8_t *a;  // bf16: sign+mantissa bytes; fp32: mantissa bytes
  const uint8_t *s;  // fp32: sign bits
};

template <int DT>
__device__ __forceinline__ void load_raw8p(const RawPtrs &p, uint32_t vl, Raw8<DT> &r) {
  if (is_fp8(DT)) {
    r.a.x = __ldg(reinterpret_cast<const uint32_t *>(p.a + vl / 2));
  } else if (DT != WC_FP32) {
    r.a = __ldg(reinterpret_cast<const uint2 *>(p.a + vl));
  } else {
    r.s = __ldg(p.s + vl / 8);
    const uint2 *m = reinterpret_cast<const uint2 *>(p.a + 3 * vl);
    r.a = __ldg(m);
    r.b = __ldg(m + 1);
    r.c = __ldg(m + 2);
  }
}

// Renormalisation of one chain whose ring starts at the 2 KiB-aligned shared
// address rs; c2 counts the bytes of words consumed.  A lane whose state fell
// below 2^16 takes the word c2 / 2 + (renormalising lanes below it): its
// address is (c2 + 2 popc(m & lt)) mod 2048 ORed onto rs, and the state takes
// the word under the same predicate that voted.
static_assert(kRing * 2 == 2048, "renorm wraps ring offsets at 2 KiB");
__device__ __forceinline__ void renorm(uint32_t &x, uint32_t &c2, uint32_t rs, uint32_t lt) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 m, t, w;\n\t"
      "setp.lt.u32 p, %0, 65536;\n\t"
      "vote.sync.ballot.b32 m, p, -1;\n\t"
      "and.b32 t, m, %3;\n\t"
      "popc.b32 t, t;\n\t"
      "mad.lo.u32 t, t, 2, %1;\n\t"
      "and.b32 t, t, 2046;\n\t"
      "or.b32 t, t, %2;\n\t"
      "ld.shared.u16 w, [t];\n\t"
      "@p prmt.b32 %0, %0, w, 0x1054;\n\t"
      "popc.b32 t, m;\n\t"
      "mad.lo.u32 %1, t, 2, %1;\n\t}"
      : "+r"(x), "+r"(c2)
      : "r"(rs), "r"(lt));
}

// One decoding step of two independent chains (chunks A and B), the table
// lookups and state updates written side by side so that each warp always
// has an independent instruction to issue while the other chain waits.
__device__ __forceinline__ void dstep2(uint32_t &xA, uint32_t &cA, uint32_t &xB, uint32_t &cB,
                                       const uint32_t *tab, uint32_t rsA, uint32_t rsB,
                                       uint8_t *tbpA, uint8_t *tbpB, uint32_t lt) {
  const uint32_t eA = tab[xA & (kProbScale - 1)];
  const uint32_t eB = tab[xB & (kProbScale - 1)];
  // f (x >> 12) + d = f ((x >> 12) - 4096) + (e >> 8), as e >> 8 = f 4096 + d
  xA = (eA >> 20) * ((xA >> kProbBits) - 4096u) + (eA >> 8);
  xB = (eB >> 20) * ((xB >> kProbBits) - 4096u) + (eB >> 8);
  *tbpA = uint8_t(eA);
  *tbpB = uint8_t(eB);
  renorm(xA, cA, rsA, lt);
  renorm(xB, cB, rsB, lt);
}

// Two full coded chunks in lock-step.  Everything arrives by value so that no
// argument lives in local memory.
// Chunk B is the one after A: its raw planes and output follow A's.
template <int DT>
__device__ __noinline__ void decode_pair(const uint8_t *payA, const uint8_t *payB, uint32_t lenA,
                                         uint32_t lenB, RawPtrs rpA, uint8_t *outA,
                                         int32_t *status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  DecSmem &s = smem();
  const uint32_t *tab = s.tab;
  const uint32_t rsA = uint32_t(__cvta_generic_to_shared(ring_ptr(warp, 0)));
  const uint32_t rsB = uint32_t(__cvta_generic_to_shared(ring_ptr(warp, 1)));
  uint8_t *tbA = s.tbuf[warp][0], *tbB = s.tbuf[warp][1];
  const uint32_t lt = lanemask_lt();
  constexpr uint32_t elem = dtype_bytes(DT);
  Ring ra{rsA, payA + kStateBytes, uint32_t(round16(lenA) - kStateBytes) >> 1, 0, 0, 0, 0};
  Ring rb{rsB, payB + kStateBytes, uint32_t(round16(lenB) - kStateBytes) >> 1, 0, 0, 0, 0};
  RawPtrs rpB;
  rpB.a = rpA.a + (DT == WC_FP32 ? 3 * kChunk : (is_fp8(DT) ? kChunk / 2 : kChunk));
  rpB.s = DT == WC_FP32 ? rpA.s + kChunk / 8 : nullptr;
  uint8_t *outB = outA + kChunk * elem;
  uint32_t xA = reinterpret_cast<const uint32_t *>(payA)[lane];
  uint32_t xB = reinterpret_cast<const uint32_t *>(payB)[lane];
  uint32_t cA = 0, cB = 0;  // bytes of words consumed
#pragma unroll
  for (int u = 0; u < int(kRing / kUnit); u++) {
    ra.issue(lane);
    rb.issue(lane);
  }
  cp_async_commit();

  constexpr uint32_t NH = kChunk / kHalf;
  // Raw planes are prefetched S half-groups ahead into S register sets used
  // in rotation; the loop is unrolled S times so each set is consumed where it
  // was loaded (no register moves that would wait on loads in flight).  fp32
  // needs 3.5x the raw bytes per value: one set, loaded a half-group ahead,
  // keeps it clear of register spills.
  constexpr int S = DT == WC_FP32 ? 1 : 4;
  Raw8<DT> pa[S], pb[S];
#pragma unroll
  for (int j = 0; j < S; j++) {
    load_raw8p<DT>(rpA, j * kHalf + 8 * lane, pa[j]);
    load_raw8p<DT>(rpB, j * kHalf + 8 * lane, pb[j]);
  }
  for (uint32_t h0 = 0; h0 < NH; h0 += S) {
#pragma unroll
    for (int j = 0; j < S; j++) {
      const uint32_t h = h0 + j;
      // The ring is checked every kSpan half-groups: up to kSpan units are
      // issued and the words of the next kSpan half-groups (at most
      // kSpan * 256; the ring keeps >= 769 requested ahead) must have landed;
      // a wait happens only when some of them are not known to have.  A wait
      // is followed by __syncwarp, so landed words are visible to every lane.
      constexpr int kSpan = S >= 2 ? 2 : 1;
      if (j % kSpan == 0) {
        const uint32_t f0A = ra.top(cA >> 1, lane), f0B = rb.top(cB >> 1, lane);
        if (kSpan == 2) {
          ra.top(cA >> 1, lane);
          rb.top(cB >> 1, lane);
        }
        cp_async_commit();
        const uint32_t needA = min((cA >> 1) + kSpan * kHalf, ra.avail);
        const uint32_t needB = min((cB >> 1) + kSpan * kHalf, rb.avail);
        if (needA > ra.landed || needB > rb.landed) {
          const int d = min(ra.depth(needA, f0A), rb.depth(needB, f0B));
          cp_async_wait_depth(d);
          ra.landed = ra.frontier(d, f0A);
          rb.landed = rb.frontier(d, f0B);
        }
        ra.shift(f0A);
        rb.shift(f0B);
        __syncwarp();
      }
#pragma unroll
      for (int t = 0; t < 8; t++)
        dstep2(xA, cA, xB, cB, tab, rsA, rsB, tbA + 32 * t + lane, tbB + 32 * t + lane, lt);
      __syncwarp();
      const uint2 eA = *reinterpret_cast<const uint2 *>(tbA + 8 * lane);
      const uint2 eB = *reinterpret_cast<const uint2 *>(tbB + 8 * lane);
      merge_store8<DT>(eA, pa[j], outA + (h * kHalf + 8 * lane) * elem);
      merge_store8<DT>(eB, pb[j], outB + (h * kHalf + 8 * lane) * elem);
      if (h + S < NH) {
        load_raw8p<DT>(rpA, (h + S) * kHalf + 8 * lane, pa[j]);
        load_raw8p<DT>(rpB, (h + S) * kHalf + 8 * lane, pb[j]);
      }
      __syncwarp();
    }
  }
  cp_async_wait<0>();
  __syncwarp();
  const uint32_t wA = (lenA - kStateBytes) >> 1, wB = (lenB - kStateBytes) >> 1;
  if (!__all_sync(0xffffffffu, xA == kStateLow) || (cA >> 1) != wA) {
    if (lane == 0) report(status, WC_ERR_CORRUPT);
  }
  if (!__all_sync(0xffffffffu, xB == kStateLow) || (cB >> 1) != wB) {
    if (lane == 0) report(status, WC_ERR_CORRUPT);
  }
}

// One chunk of any kind (raw, single-symbol, coded, ragged).
template <int DT>
__device__ __noinline__ void decode_one(const ItemView &v, const DecItem &it, const ChunkView &c,
                           uint64_t k, int slot, int32_t *status) {
  DecSmem &s = smem();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = lanemask_lt();
  const Layout &L = v.L;
  constexpr uint32_t elem = dtype_bytes(DT);
  const uint64_t vg0 = k * kChunk;
  const uint32_t nsym = c.nsym;
  const uint32_t nhalf = (nsym + kHalf - 1) / kHalf;
  uint8_t *tb = s.tbuf[warp][slot];

  int mode = c.raw ? 0 : (s.single_sym >= 0 ? 1 : 2);
  uint32_t x = 0, cons = 0;
  const uint16_t *rbuf = ring_ptr(warp, slot);
  Ring r{uint32_t(__cvta_generic_to_shared(rbuf)), c.pay + kStateBytes, 0, 0, 0, 0, 0};
  if (mode == 1) {
    // single-symbol table: coding never moves a state and never emits a word
    x = reinterpret_cast<const uint32_t *>(c.pay)[lane];
    if (!__all_sync(0xffffffffu, x == kStateLow) || c.len != kStateBytes) {
      if (lane == 0) report(status, WC_ERR_CORRUPT);
      return;
    }
  } else if (mode == 2) {
    x = reinterpret_cast<const uint32_t *>(c.pay)[lane];
    r.avail = uint32_t(round16(c.len) - kStateBytes) >> 1;
#pragma unroll
    for (int u = 0; u < int(kRing / kUnit); u++) r.issue(lane);
    cp_async_commit();
  }
  const uint32_t single_e = uint32_t(s.single_sym) * 0x01010101u;
  for (uint32_t h = 0; h < nhalf; h++) {
    const uint32_t hb = h * kHalf;
    const bool full = hb + kHalf <= nsym;
    if (mode == 2) {
      const int d = r.top_up(cons, lane);
      cp_async_commit();
      cp_async_wait_depth(d);
      __syncwarp();
      if (full) {
#pragma unroll
        for (int t = 0; t < 8; t++) dstep(x, cons, s.tab, rbuf, tb + 32 * t + lane, lt);
      } else {
        const uint32_t steps = (nsym - hb + 31) / 32;
        for (uint32_t t = 0; t < steps; t++) {
          const bool valid = hb + 32 * t + lane < nsym;
          uint32_t e = 0;
          if (valid) {
            e = s.tab[x & (kProbScale - 1)];
            x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
          }
          const bool rn = valid && x < kStateLow;
          const uint32_t m = __ballot_sync(0xffffffffu, rn);
          const uint32_t w = rbuf[(cons + __popc(m & lt)) & (kRing - 1)];
          if (rn) x = __byte_perm(x, w, 0x1054);
          cons += __popc(m);
          tb[32 * t + lane] = uint8_t(e);
        }
      }
      __syncwarp();
    }
    const uint32_t vl = hb + 8 * lane;  // this lane's first value in the chunk
    if (full) {
      uint2 e8;
      if (mode == 0) e8 = __ldg(reinterpret_cast<const uint2 *>(c.pay + vl));
      else if (mode == 1) e8 = make_uint2(single_e, single_e);
      else e8 = *reinterpret_cast<const uint2 *>(tb + 8 * lane);
      Raw8<DT> rr;
      load_raw8<DT>(it.cont, L, vg0 + vl, rr);
      merge_store8<DT>(e8, rr, c.out + uint64_t(vl) * elem);
    } else {
      for (uint32_t j = 0; j < 8 && vl + j < nsym; j++) {
        uint32_t e;
        if (mode == 0) e = c.pay[vl + j];
        else if (mode == 1) e = uint32_t(s.single_sym);
        else e = tb[8 * lane + j];
        merge_store1<DT>(e, it.cont, L, vg0 + vl + j, c.out + uint64_t(vl + j) * elem);
      }
    }
    if (mode == 2) __syncwarp();
  }
  if (mode == 2) {
    cp_async_wait<0>();
    __syncwarp();
    if (!__all_sync(0xffffffffu, x == kStateLow) || cons != ((c.len - kStateBytes) >> 1)) {
      if (lane == 0) report(status, WC_ERR_CORRUPT);
    }
  }
}

// ---------------------------------------------------------------------------
// Build the decoding table of item ii (whole block).
__device__ __noinline__ void build_table(const DecItem &it, int ii, int32_t *status) {
  DecSmem &s = smem();
  const int tid = threadIdx.x;
  __syncthreads();  // all warps are done with the previous table and rings
  uint32_t *sfreq = reinterpret_cast<uint32_t *>(ring_ptr(0, 0));
  uint32_t *scum = sfreq + 256;
  const uint16_t *f16 = reinterpret_cast<const uint16_t *>(it.cont + kFreqOffset);
  const uint32_t f = f16[tid];
  const uint64_t sum = block_sum_u64<kDecThreads>(f, s.red);
  const uint64_t cum = block_excl_scan_u64<kDecThreads>(f, s.red);
  const uint64_t single = block_max_u64<kDecThreads>(f == kProbScale ? uint64_t(tid) + 1 : 0, s.red);
  sfreq[tid] = f;
  scum[tid] = uint32_t(cum);
  const bool ok = sum == kProbScale;
  __syncthreads();
  if (ok && single == 0) {
    constexpr uint32_t per = kProbScale / kDecThreads;  // 16 slots per thread
    const uint32_t j0 = uint32_t(tid) * per;
    uint32_t lo = 0, hi = 255;  // last symbol with cum <= j0
    while (lo < hi) {
      uint32_t mid = (lo + hi + 1) >> 1;
      if (scum[mid] <= j0) lo = mid; else hi = mid - 1;
    }
    uint32_t sym = lo;
    for (uint32_t j = j0; j < j0 + per; j++) {
      while (j >= scum[sym] + sfreq[sym]) sym++;
      s.tab[j] = sym | ((j - scum[sym]) << 8) | (sfreq[sym] << 20);
    }
  }
  if (tid == 0) {
    s.cur_item = ii;
    s.tab_ok = ok;
    s.single_sym = single ? int(single - 1) : -1;
    if (!ok) report(status, WC_ERR_CORRUPT);
  }
  __syncthreads();
}

template <int DT>
__device__ __forceinline__ void decode_warp_chunks(const ItemView &v, const DecItem &it,
                                                   uint64_t kA, uint64_t kend, int32_t *status) {
  DecSmem &s = smem();
  const int lane = threadIdx.x & 31;
  if (kA >= kend) return;
  const ChunkView A = view_chunk<DT>(it, v, kA);
  const bool hasB = kA + 1 < kend;
  ChunkView B;
  if (hasB) B = view_chunk<DT>(it, v, kA + 1);
  if (!A.ok || (hasB && !B.ok)) {
    if (lane == 0) report(status, WC_ERR_CORRUPT);
    return;
  }
  if (hasB && s.single_sym < 0 && !A.raw && !B.raw && A.nsym == kChunk && B.nsym == kChunk) {
    const Layout &L = v.L;
    const uint64_t vgA = kA * kChunk;
    RawPtrs rpA;
    if (is_fp8(DT)) {
      rpA.a = it.cont + L.off_raw + vgA / 2;
      rpA.s = nullptr;
    } else if (DT != WC_FP32) {
      rpA.a = it.cont + L.off_raw + vgA;
      rpA.s = nullptr;
    } else {
      rpA.a = it.cont + L.off_mant + 3 * vgA;
      rpA.s = it.cont + L.off_raw + vgA / 8;
    }
    decode_pair<DT>(A.pay, B.pay, A.len, B.len, rpA, A.out, status);
    return;
  }
  decode_one<DT>(v, it, A, kA, 0, status);
  if (hasB) decode_one<DT>(v, it, B, kA + 1, 1, status);
}

__global__ void __launch_bounds__(kDecThreads, 4) k_decode(const __grid_constant__ DecParams p) {
  DecSmem &s = smem();
  const int tid = threadIdx.x, warp = tid >> 5;
  int32_t *status = p.status;

  // prologue: chunks per item (one item per thread); the group size: 16
  // chunks (8 warps x 2, decoded in lock-step) when the launch has enough
  // for every block; with more chunks than warps, the even number that
  // spreads them over all blocks; with fewer, one chunk a warp (a chunk is a
  // chain of dependent steps: few chunks go faster one chain per warp) and as
  // many a block as spread them; groups per item -> prefix
  uint64_t cnt = 0;
  if (uint32_t(tid) < p.count) {
    const ItemView v = view_item(p.items[tid]);
    if (v.ok) cnt = v.cnt;
    else if (blockIdx.x == 0) report(status, v.err);
  }
  const uint64_t chunks = block_sum_u64<kDecThreads>(cnt, s.red);
  const bool single = chunks <= uint64_t(kDecWarps) * gridDim.x;
  uint32_t group;
  if (single) {
    const uint64_t per_block = (chunks + gridDim.x - 1) / gridDim.x;
    group = uint32_t(per_block < 1 ? 1 : per_block);  // <= kDecWarps
  } else {
    const uint64_t per_block = (chunks + 2 * uint64_t(gridDim.x) - 1) / (2 * uint64_t(gridDim.x));  // pairs
    group = uint32_t(per_block >= kDecGroup / 2 ? kDecGroup : 2 * per_block);
  }
  const uint32_t g = uint32_t((cnt + group - 1) / group);
  const uint64_t ex = block_excl_scan_u64<kDecThreads>(g, s.red);
  s.gpre[tid] = uint32_t(ex);
  if (tid == kDecThreads - 1) s.gpre[kMaxItems] = uint32_t(ex) + g;
  if (tid == 0) s.cur_item = -1;
  __syncthreads();
  const uint32_t total = s.gpre[kMaxItems];

  for (;;) {
    __syncthreads();  // every thread has read the previous group's number
    if (tid == 0) s.next_grp = atomicAdd(p.queue, 1u);
    __syncthreads();
    const uint32_t grp = s.next_grp;
    if (grp >= total) break;
    uint32_t lo = 0, hi = p.count - 1;  // last item with gpre <= grp
    while (lo < hi) {
      uint32_t mid = (lo + hi + 1) >> 1;
      if (s.gpre[mid] <= grp) lo = mid; else hi = mid - 1;
    }
    const int ii = int(lo);
    const DecItem &it = p.items[ii];
    const ItemView v = view_item(it);
    if (ii != s.cur_item) build_table(it, ii, status);
    if (!s.tab_ok) continue;
    if (uint32_t(single ? warp : 2 * warp) >= group) continue;  // no chunk for this warp in a small group
    const uint64_t kA = v.first + uint64_t(grp - s.gpre[ii]) * group + (single ? warp : 2 * warp);
    const uint64_t kend = single ? min(v.first + v.cnt, kA + 1) : v.first + v.cnt;
    if (v.dtype == WC_BF16) decode_warp_chunks<WC_BF16>(v, it, kA, kend, status);
    else if (v.dtype == WC_FP16) decode_warp_chunks<WC_FP16>(v, it, kA, kend, status);
    else if (v.dtype == WC_FP8E4M3) decode_warp_chunks<WC_FP8E4M3>(v, it, kA, kend, status);
    else if (v.dtype == WC_FP8E5M2) decode_warp_chunks<WC_FP8E5M2>(v, it, kA, kend, status);
    else decode_warp_chunks<WC_FP32>(v, it, kA, kend, status);
  }
}

// Per device, before the first launch: allow the kernel its dynamic shared
// memory and return how many blocks fit on one SM.
int decode_blocks_per_sm() {
  if (cudaFuncSetAttribute(k_decode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(sizeof(DecSmem))) != cudaSuccess)
    return 0;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_decode, kDecThreads, sizeof(DecSmem)) !=
      cudaSuccess)
    return 0;
  return nb;
}

// The launches' group counters: a library-held array of slots, one per
// launch in rotation, each zeroed on the launch's stream before it runs, so
// that calls overlapping on other streams (up to kQueueSlots of them) never
// share one.
constexpr uint32_t kQueueSlots = 4096;
__device__ uint32_t g_dec_queue[kQueueSlots];

// Device address of g_dec_queue on the current device, cached per device
// together with the context it belongs to.
static uint32_t *queue_base() {
  struct Entry {
    uint32_t *addr = nullptr;
    unsigned long long ctx = 0;
  };
  static std::mutex mu;
  static Entry cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  Entry &c = cache[dev];
  const unsigned long long ctx = current_context_id();
  if (c.addr == nullptr || ctx == 0 || c.ctx != ctx) {
    void *a = nullptr;
    if (cudaGetSymbolAddress(&a, g_dec_queue) != cudaSuccess || a == nullptr) return nullptr;
    c.addr = static_cast<uint32_t *>(a);
    c.ctx = current_context_id();
  }
  return c.addr;
}

cudaError_t launch_decode(DecParams &p, int grid, cudaStream_t s) {
  static std::atomic<uint32_t> next_slot{0};
  uint32_t *base = queue_base();
  if (base == nullptr) return cudaErrorInvalidSymbol;
  p.queue = base + next_slot.fetch_add(1u) % kQueueSlots;
  cudaError_t e = cudaMemsetAsync(p.queue, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  k_decode<<<grid, kDecThreads, sizeof(DecSmem), s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
