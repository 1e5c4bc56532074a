// wc12_plan.cuh -- layout of the serving plan of a Split12 container
// (include/wc_split12.h, wc12_plan): the container's exceptions grouped by
// the tiles wc12_linear works in, 128 weight rows by 64 values of K, so that
// a CTA finds its tile's exceptions as one range of the plan.  Shared by the
// plan builder (k_split12_plan.cu) and the linear layer (k_split12_linear.cu).
//
//   0   u32 magic "W12P"   u32 version 1   u32 N   u32 K
//   16  u64 ne (the container's exceptions)   24 u64 buckets = N/128 * K/64
//   32  u32 start[buckets + 1]: bucket (row block b, stage s) is
//       b * (K / 64) + s; its entries are [start[i], start[i + 1])
//   off_ent (16-byte aligned)  u32 entry[ne]: column in the stage (bits
//       0-5), row in the block (bits 6-12), the exception's high byte (bits
//       16-23); any order within a bucket
#pragma once

#include <cstdint>

#include "wc_split12.cuh"

namespace wc12p {

constexpr uint32_t kMagic = 0x50323157u;  // "W12P"
constexpr uint32_t kRows = 128;           // weight rows of a tile
constexpr uint32_t kValues = 64;          // values of K of a tile (a stage)
constexpr uint64_t kStartOff = 32;

struct PlanLay {
  uint64_t buckets, off_ent, total;
};

__host__ __device__ inline PlanLay plan_lay(uint32_t N, uint32_t K, uint64_t ne) {
  PlanLay P;
  P.buckets = uint64_t(N / kRows) * (K / kValues);
  P.off_ent = wc12::r16(kStartOff + 4 * (P.buckets + 1));
  P.total = wc12::r16(P.off_ent + 4 * ne);
  return P;
}

__host__ __device__ inline uint32_t pack_entry(uint32_t col_in_stage, uint32_t row_in_block, uint32_t high) {
  return col_in_stage | (row_in_block << 6) | (high << 16);
}

}  // namespace wc12p
