// k_decode.cu -- decoder: rANS decode of the exponent chunks fused with the
// re-merge of the planes into the original bits ("PTWM" How it works 1-2 run
// backwards; "SMEF" pass3_streams.py merge_streams).
//
// Persistent grid.  Work is split into groups of kDecWarps consecutive chunks
// of one tensor; a block takes groups blockIdx.x, + gridDim.x, ...  A block
// stages its tensor's 4096-slot decoding table in shared memory (entry =
// symbol | (slot - cum) << 8 | f << 20), then each warp decodes one chunk:
//   slot = x & 4095; e = tab[slot]; x = f (x >> 12) + (slot - cum);
//   if x < 2^16: x = x << 16 | next word
// where the lanes needing a word at a step take consecutive words in lane
// order (__ballot_sync / __popc), from a per-warp shared-memory ring that
// cp.async keeps filled with 16-byte loads of the chunk's word stream.  Every
// 16 steps the warp has 512 exponent bytes; they are transposed through shared
// memory so that each lane holds 16 consecutive ones, merged with the matching
// raw-plane bytes, and written with 16-byte stores.
//
// Everything read from the container is checked before use (header fields
// against the layout implied by n, the table sum, each chunk's offset pair and
// length); a decoded chunk must end with every lane at 2^16 and every word
// consumed.  Failures store a wc_status code in *status and skip the chunk.
// No loop waits on another block; each wait is on this warp's own copies.
#include "wc_block.cuh"
#include "wc_format.cuh"

namespace wc {

constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kRing = 1024;  // words per warp (4 units of 256)
constexpr uint32_t kUnit = 256;   // words per cp.async round (32 lanes x 16 B)

struct DecSmem {
  uint32_t tab[kProbScale];                      // 16 KiB
  __align__(16) uint16_t ring[kDecWarps][kRing];  // also holds freq/cum while a table is built
  __align__(16) uint8_t tbuf[kDecWarps][kGroupValues];
  uint32_t gpre[kMaxItems + 1];
  uint64_t red[kDecThreads / 32 + 1];
  int cur_item;
  int tab_ok;
  int single_sym;
};

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
__device__ ItemView view_item(const DecItem &it) {
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
  if (dtype != WC_BF16 && dtype != WC_FP32) return v;
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
  const uint64_t elem = dtype == WC_BF16 ? 2 : 4;
  const uint64_t vals = v.cnt == 0 ? 0
                        : (v.first + v.cnt == L.nc ? n - v.first * kChunk : v.cnt * kChunk);
  if (vals * elem > it.out_cap || (vals > 0 && it.out == nullptr)) { v.err = WC_ERR_CAPACITY; return v; }
  v.ok = true;
  v.err = WC_OK;
  return v;
}

// ---------------------------------------------------------------------------
// raw-plane bytes of 16 values and the merge
template <int DT>
struct Raw {
  uint4 a;            // bf16: 16 sign+mantissa bytes; fp32: mantissa words 0..3
  uint4 b, c;         // fp32: mantissa words 4..11
  uint32_t sbits;     // fp32: 16 sign bits
};

template <int DT>
__device__ __forceinline__ void load_raw(const uint8_t *cont, const Layout &L, uint64_t vg, uint32_t nv,
                                         Raw<DT> &r) {
  if (DT == WC_BF16) {
    const uint8_t *s = cont + L.off_raw + vg;
    if (nv == 16) {
      r.a = ld_nc_v4(s);
    } else {
      uint32_t w[4] = {0, 0, 0, 0};
      for (uint32_t j = 0; j < nv; j++) {
        uint32_t byte = s[j];
#pragma unroll
        for (int q = 0; q < 4; q++)
          if (q == int(j >> 2)) w[q] |= byte << (8 * (j & 3));
      }
      r.a = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    const uint8_t *ss = cont + L.off_raw + vg / 8;
    const uint8_t *ms = cont + L.off_mant + 3 * vg;
    if (nv == 16) {
      r.sbits = *reinterpret_cast<const uint16_t *>(ss);
      r.a = ld_nc_v4(ms);
      r.b = ld_nc_v4(ms + 16);
      r.c = ld_nc_v4(ms + 32);
    } else {
      r.sbits = ss[0] | (nv > 8 ? uint32_t(ss[1]) << 8 : 0u);
      uint32_t w[12];
#pragma unroll
      for (int q = 0; q < 12; q++) w[q] = 0;
      for (uint32_t j = 0; j < 3 * nv; j++) {
        uint32_t byte = ms[j];
#pragma unroll
        for (int q = 0; q < 12; q++)
          if (q == int(j >> 2)) w[q] |= byte << (8 * (j & 3));
      }
      r.a = make_uint4(w[0], w[1], w[2], w[3]);
      r.b = make_uint4(w[4], w[5], w[6], w[7]);
      r.c = make_uint4(w[8], w[9], w[10], w[11]);
    }
  }
}

// bf16 pair from exponent word ew and sign+mantissa word sw (bytes 2h, 2h+1):
// b = sm + 128 e + 255 (sm & 0x80)   (= s << 15 | e << 7 | m)
__device__ __forceinline__ uint32_t merge_bf16_pair(uint32_t ew, uint32_t sw, int h) {
  const uint32_t sel = h ? 0x4342u : 0x4140u;
  const uint32_t eh = __byte_perm(ew, 0, sel);
  const uint32_t sh = __byte_perm(sw, 0, sel);
  return sh + (eh << 7) + (sh & 0x00800080u) * 255u;
}

template <int DT>
__device__ __forceinline__ void merge_store(uint4 e, const Raw<DT> &r, uint8_t *dst, uint32_t nv) {
  if (DT == WC_BF16) {
    uint32_t o[8];
    o[0] = merge_bf16_pair(e.x, r.a.x, 0); o[1] = merge_bf16_pair(e.x, r.a.x, 1);
    o[2] = merge_bf16_pair(e.y, r.a.y, 0); o[3] = merge_bf16_pair(e.y, r.a.y, 1);
    o[4] = merge_bf16_pair(e.z, r.a.z, 0); o[5] = merge_bf16_pair(e.z, r.a.z, 1);
    o[6] = merge_bf16_pair(e.w, r.a.w, 0); o[7] = merge_bf16_pair(e.w, r.a.w, 1);
    if (nv == 16) {
      st_cs_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
      st_cs_v4(dst + 16, make_uint4(o[4], o[5], o[6], o[7]));
    } else {
      uint16_t *d16 = reinterpret_cast<uint16_t *>(dst);
      for (uint32_t j = 0; j < nv; j++) {
        uint32_t word = 0;
#pragma unroll
        for (int q = 0; q < 8; q++)
          if (q == int(j >> 1)) word = o[q];
        d16[j] = uint16_t(word >> (16 * (j & 1)));
      }
    }
  } else {
    const uint32_t mw[12] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w,
                             r.c.x, r.c.y, r.c.z, r.c.w};
    const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const uint32_t w0 = mw[3 * q], w1 = mw[3 * q + 1], w2 = mw[3 * q + 2];
      const uint32_t m[4] = {w0 & 0x7FFFFFu, __funnelshift_r(w0, w1, 24) & 0x7FFFFFu,
                             __funnelshift_r(w1, w2, 16) & 0x7FFFFFu, (w2 >> 8) & 0x7FFFFFu};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const uint32_t ex = (ew[q] >> (8 * j)) & 0xFFu;
        const uint32_t sg = (r.sbits >> (4 * q + j)) & 1u;
        o[4 * q + j] = (sg << 31) | (ex << 23) | m[j];
      }
    }
    if (nv == 16) {
#pragma unroll
      for (int q = 0; q < 4; q++)
        st_cs_v4(dst + 16 * q, make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]));
    } else {
      uint32_t *d32 = reinterpret_cast<uint32_t *>(dst);
#pragma unroll
      for (int q = 0; q < 16; q++)
        if (uint32_t(q) < nv) d32[q] = o[q];
    }
  }
}

// ---------------------------------------------------------------------------
template <int DT>
__device__ void decode_chunk(DecSmem &s, const DecItem &it, const ItemView &v, uint64_t k,
                             int32_t *status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const Layout &L = v.L;
  const uint8_t *cont = it.cont;
  const uint32_t nsym = chunk_nsym(v.n, k);
  const uint64_t *choff = reinterpret_cast<const uint64_t *>(cont + L.off_chunk_off);
  const uint32_t *chlen = reinterpret_cast<const uint32_t *>(cont + L.off_chunk_len);
  const uint64_t exp_bytes = reinterpret_cast<const uint64_t *>(cont)[6];
  const uint64_t o0 = choff[k], o1 = choff[k + 1];
  const uint32_t len = chlen[k];
  const bool raw = len == nsym;
  const bool coded = len >= kStateBytes && len < nsym && (len & 1u) == 0;
  bool ok = (raw || coded) && o0 <= o1 && o1 - o0 == round16(len) && o1 <= exp_bytes &&
            (k != 0 || o0 == 0) && (k + 1 != L.nc || o1 == exp_bytes);
  if (!ok) {
    if (lane == 0) report(status, WC_ERR_CORRUPT);
    return;
  }
  constexpr uint32_t elem = DT == WC_BF16 ? 2 : 4;
  const uint8_t *pay = cont + L.off_exp + o0;
  uint8_t *outc = it.out + (k - v.first) * kChunk * elem;
  const int ngroups = int((nsym + kGroupValues - 1) / kGroupValues);
  auto lane_nv = [&](int G) -> uint32_t {
    int64_t r = int64_t(nsym) - (int64_t(G) * kGroupValues + 16 * lane);
    return r <= 0 ? 0u : (r >= 16 ? 16u : uint32_t(r));
  };

  if (raw || s.single_sym >= 0) {
    uint4 ec = make_uint4(0, 0, 0, 0);
    if (!raw) {
      // single-symbol table: coding never moves a state and never emits a word
      const uint32_t x = reinterpret_cast<const uint32_t *>(pay)[lane];
      const bool good = __all_sync(0xffffffffu, x == kStateLow) && len == kStateBytes;
      if (!good) {
        if (lane == 0) report(status, WC_ERR_CORRUPT);
        return;
      }
      const uint32_t b = uint32_t(s.single_sym) * 0x01010101u;
      ec = make_uint4(b, b, b, b);
    }
    for (int G = 0; G < ngroups; G++) {
      const uint32_t nv = lane_nv(G);
      if (nv == 0) continue;
      const uint32_t vl = uint32_t(G) * kGroupValues + 16 * lane;
      Raw<DT> r;
      load_raw<DT>(cont, L, k * kChunk + vl, nv, r);
      const uint4 e = raw ? ld_nc_v4(pay + vl) : ec;  // raw payload is padded to 16
      merge_store<DT>(e, r, outc + uint64_t(vl) * elem, nv);
    }
    return;
  }

  // ---- rANS chunk
  const uint32_t lt = lanemask_lt();
  uint32_t x = reinterpret_cast<const uint32_t *>(pay)[lane];
  const uint32_t w = (len - kStateBytes) >> 1;
  const uint8_t *wsrc = pay + kStateBytes;
  const uint32_t wavail = uint32_t(round16(len) - kStateBytes) >> 1;  // readable words
  uint16_t *ring = s.ring[warp];
  uint8_t *tb = s.tbuf[warp];
  const uint32_t *tab = s.tab;
  uint32_t req = 0, cons = 0;

  auto issue = [&]() {
    const uint32_t j0 = req + 8 * lane;
    if (j0 < wavail) cp_async16(ring + (j0 & (kRing - 1)), wsrc + 2 * j0, 16);
    else cp_async16(ring + (j0 & (kRing - 1)), wsrc, 0);  // zero fill, reads nothing
    req += kUnit;
  };
#pragma unroll
  for (int u = 0; u < int(kRing / kUnit); u++) issue();
  cp_async_commit();

  for (int G = 0; G < ngroups; G++) {
    const uint32_t before = req;
    while (req < wavail && req + kUnit <= (cons & ~(kUnit - 1)) + kRing) issue();
    cp_async_commit();
    const uint32_t need = min(cons + kGroupValues, wavail);
    if (before >= need) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncwarp();

    const uint32_t nv = lane_nv(G);
    const uint32_t vl = uint32_t(G) * kGroupValues + 16 * lane;
    Raw<DT> r;
    if (nv) load_raw<DT>(cont, L, k * kChunk + vl, nv, r);

    const uint32_t gbase = uint32_t(G) * kGroupValues;
    if (gbase + kGroupValues <= nsym) {
#pragma unroll
      for (int t = 0; t < int(kStepsPerGroup); t++) {
        const uint32_t e = tab[x & (kProbScale - 1)];
        x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
        const bool rn = x < kStateLow;
        const uint32_t m = __ballot_sync(0xffffffffu, rn);
        if (rn) x = (x << 16) | ring[(cons + __popc(m & lt)) & (kRing - 1)];
        cons += __popc(m);
        tb[32 * t + lane] = uint8_t(e);
      }
    } else {
      const int steps = int((nsym - gbase + 31) / 32);
      for (int t = 0; t < steps; t++) {
        const bool valid = gbase + 32 * t + lane < nsym;
        uint32_t e = 0;
        if (valid) {
          e = tab[x & (kProbScale - 1)];
          x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
        }
        const bool rn = valid && x < kStateLow;
        const uint32_t m = __ballot_sync(0xffffffffu, rn);
        if (rn) x = (x << 16) | ring[(cons + __popc(m & lt)) & (kRing - 1)];
        cons += __popc(m);
        tb[32 * t + lane] = uint8_t(e);
      }
    }
    __syncwarp();
    if (nv) {
      const uint4 e = *reinterpret_cast<const uint4 *>(tb + 16 * lane);
      merge_store<DT>(e, r, outc + uint64_t(vl) * elem, nv);
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncwarp();
  const bool good = __all_sync(0xffffffffu, x == kStateLow) && cons == w;
  if (!good && lane == 0) report(status, WC_ERR_CORRUPT);
}

// ---------------------------------------------------------------------------
// Build the decoding table of item ii (whole block).
__device__ void build_table(DecSmem &s, const DecItem &it, int ii, int32_t *status) {
  const int tid = threadIdx.x;
  __syncthreads();  // all warps are done with the previous table and rings
  uint32_t *sfreq = reinterpret_cast<uint32_t *>(&s.ring[0][0]);
  uint32_t *scum = sfreq + 256;
  const uint16_t *f16 = reinterpret_cast<const uint16_t *>(it.cont + kFreqOffset);
  const uint32_t f0 = f16[2 * tid], f1 = f16[2 * tid + 1];
  const uint64_t sum = block_sum_u64<kDecThreads>(f0 + f1, s.red);
  const uint64_t ex = block_excl_scan_u64<kDecThreads>(f0 + f1, s.red);
  uint64_t single = 0;
  if (f0 == kProbScale) single = 2 * tid + 1;
  if (f1 == kProbScale) single = 2 * tid + 2;
  single = block_max_u64<kDecThreads>(single, s.red);
  sfreq[2 * tid] = f0;
  sfreq[2 * tid + 1] = f1;
  scum[2 * tid] = uint32_t(ex);
  scum[2 * tid + 1] = uint32_t(ex) + f0;
  const bool ok = sum == kProbScale;
  __syncthreads();
  if (ok && single == 0) {
    // thread t fills slots [32 t, 32 t + 32)
    const uint32_t j0 = uint32_t(tid) * (kProbScale / kDecThreads);
    uint32_t lo = 0, hi = 255;  // last symbol with cum <= j0
    while (lo < hi) {
      uint32_t mid = (lo + hi + 1) >> 1;
      if (scum[mid] <= j0) lo = mid; else hi = mid - 1;
    }
    uint32_t sym = lo;
    for (uint32_t j = j0; j < j0 + kProbScale / kDecThreads; j++) {
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

__global__ void __launch_bounds__(kDecThreads, 8) k_decode(const __grid_constant__ DecParams p) {
  __shared__ DecSmem s;
  const int tid = threadIdx.x, warp = tid >> 5;
  int32_t *status = p.status;

  // prologue: groups per item -> prefix (two items per thread)
  uint32_t g2[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const uint32_t i = 2 * tid + h;
    if (i < p.count) {
      const ItemView v = view_item(p.items[i]);
      if (v.ok) g2[h] = uint32_t((v.cnt + kDecWarps - 1) / kDecWarps);
      else if (blockIdx.x == 0) report(status, v.err);
    }
  }
  const uint64_t ex = block_excl_scan_u64<kDecThreads>(g2[0] + g2[1], s.red);
  if (2 * tid < kMaxItems) s.gpre[2 * tid] = uint32_t(ex);
  if (2 * tid + 1 < kMaxItems) s.gpre[2 * tid + 1] = uint32_t(ex) + g2[0];
  if (tid == kDecThreads - 1) s.gpre[kMaxItems] = uint32_t(ex) + g2[0] + g2[1];
  if (tid == 0) s.cur_item = -1;
  __syncthreads();
  const uint32_t total = s.gpre[kMaxItems];

  for (uint32_t grp = blockIdx.x; grp < total; grp += gridDim.x) {
    uint32_t lo = 0, hi = p.count - 1;  // last item with gpre <= grp
    while (lo < hi) {
      uint32_t mid = (lo + hi + 1) >> 1;
      if (s.gpre[mid] <= grp) lo = mid; else hi = mid - 1;
    }
    const int ii = int(lo);
    const DecItem &it = p.items[ii];
    const ItemView v = view_item(it);
    if (ii != s.cur_item) build_table(s, it, ii, status);
    if (!s.tab_ok) continue;
    const uint64_t k = v.first + uint64_t(grp - s.gpre[ii]) * kDecWarps + warp;
    if (k >= v.first + v.cnt) continue;
    if (v.dtype == WC_BF16) decode_chunk<WC_BF16>(s, it, v, k, status);
    else decode_chunk<WC_FP32>(s, it, v, k, status);
  }
}

int decode_blocks_per_sm() {
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_decode, kDecThreads, 0) != cudaSuccess)
    return 1;
  return nb > 0 ? nb : 1;
}

cudaError_t launch_decode(const DecParams &p, int grid, cudaStream_t s) {
  k_decode<<<grid, kDecThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace wc
