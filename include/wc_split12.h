/*
 * wc_split12.h -- the Split12 serving format for bf16 weights, in libwc.so.
 *
 * "weight-compression" README: Split12 splits bf16 into its two bytes,
 * rebuilds the high byte from a codebook and keeps the low byte raw (24.967 %
 * smaller on a 753B model).  Read as 12 bits a value: a 4-bit index into the
 * tensor's 16-entry codebook of high bytes plus the raw low byte; values
 * whose high byte the codebook misses are listed as exceptions.  It decodes
 * with a few instructions per value, so it is the format a GEMM can expand
 * in its prologue; the rANS container of wc.h stays the smaller storage
 * format.
 *
 * Container "W12C" (little-endian; sections 16-byte aligned, zero padding):
 *   0   "W12C", u16 version 1, u8 dtype 1 (bf16), u8 K (codebook entries)
 *   8   u64 n
 *   16  u32 chunk values 65536, u32 nc = ceil(n / 65536)
 *   24  u64 ne (exceptions)
 *   32  u64 off_idx, u64 off_lo, u64 off_exc, u64 total bytes
 *   64  u8 codebook[16]: the K most frequent high bytes (b >> 8) of the
 *       tensor, ties to the smaller byte, ascending; entries >= K are 0
 *   80  u64 exc_off[nc + 1]: first exception of each chunk; exc_off[nc] = ne
 *   off_idx = round16(80 + 8 (nc + 1)): ceil(n / 2) bytes of 4-bit indices,
 *       value i in byte i / 2, low nibble for even i; 0 for an exception
 *   off_lo = round16(off_idx + ceil(n / 2)): the n low bytes (b & 0xFF)
 *   off_exc = round16(off_lo + n): u16 position of each exception within its
 *       chunk, ascending within the chunk, chunk by chunk
 *   off_exc + round16(2 ne): the exceptions' u8 high bytes
 *   total = off_exc + round16(2 ne) + round16(ne)
 * Exactly one container is correct for an input.
 *
 * Conventions are those of wc.h: device pointers, caller-owned buffers, no
 * allocation, no synchronisation, work queued on `stream`; argument errors
 * return synchronously, container problems go to *d_status.
 */
#ifndef WC_SPLIT12_H
#define WC_SPLIT12_H

#include <stdint.h>

#include "wc.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Largest container for n values (at most 15n/16 of them can be exceptions:
 * the 16 most frequent high bytes hold at least n/16 of the values). */
WC_API uint64_t wc12_encode_bound(uint64_t n);

/* Device scratch wc12_encode needs for n values (2,560 B plus 1 KiB per
 * 65,536-value chunk). */
WC_API uint64_t wc12_scratch_bytes(uint64_t n);

/* Encode n bf16 values (d_in, 16-byte aligned) into d_out (16-byte aligned,
 * out_cap >= wc12_encode_bound(n)); the container's size goes to the device
 * u64 *d_out_size.  d_scratch: 16-byte aligned, wc12_scratch_bytes(n) bytes.
 * Returns WC_OK, WC_ERR_INVALID_ARG, WC_ERR_CAPACITY or WC_ERR_CUDA. */
WC_API int32_t wc12_encode(const void *d_in, uint64_t n, void *d_out, uint64_t out_cap,
                           void *d_scratch, uint64_t scratch_cap, uint64_t *d_out_size,
                           void *stream);

/* Header of a container of `bytes` bytes, read from a host copy of its first
 * 64 bytes (h_cont): n, exceptions, codebook entries.  Checks what
 * wc12_decode checks of the header and layout (magic, version, dtype, K,
 * chunk size and count, section offsets, total <= bytes; fewer than 96 bytes
 * is corrupt).  Returns WC_OK, WC_ERR_INVALID_ARG (null pointer) or
 * WC_ERR_CORRUPT.  Host only. */
WC_API int32_t wc12_read_header(const void *h_cont, uint64_t bytes, uint64_t *n, uint64_t *ne,
                                uint32_t *k);

/* Many tensors in one call: one launch per encoder kernel for the whole
 * list (in groups of 256 tensors), each item exactly as wc12_encode's
 * arguments.  All checks are made before anything is launched. */
typedef struct {
  const void *in;      /* n bf16 values, 16-byte aligned (may be NULL if n == 0) */
  uint64_t n;
  void *out;           /* container, 16-byte aligned, out_cap >= wc12_encode_bound(n) */
  uint64_t out_cap;
  void *scratch;       /* 16-byte aligned, scratch_cap >= wc12_scratch_bytes(n) */
  uint64_t scratch_cap;
  uint64_t *out_size;  /* device u64, 8-byte aligned: the container's size */
} wc12_encode_item;
WC_API int32_t wc12_encode_batch(const wc12_encode_item *items, uint32_t count, void *stream);

/* Decode a container (d_cont, cont_bytes, 16-byte aligned) into out_cap bytes
 * at d_out (16-byte aligned).  *d_status (device i32, set to 0 by the caller)
 * receives WC_ERR_CORRUPT for a bad header, offset table, index >= K or
 * exception position, WC_ERR_CAPACITY if 2n > out_cap; the output is then
 * unspecified but nothing outside [d_out, d_out + out_cap) is written.
 * Returns WC_OK, WC_ERR_INVALID_ARG or WC_ERR_CUDA. */
WC_API int32_t wc12_decode(const void *d_cont, uint64_t cont_bytes, void *d_out, uint64_t out_cap,
                           int32_t *d_status, void *stream);

/* Many containers in one launch (in groups of 256): item i decodes cont
 * (16-byte aligned, cont_bytes) into out (16-byte aligned, room for 2 n
 * bytes), where n is the number of values the caller expects; a container
 * whose header gives another n is reported as WC_ERR_CORRUPT.  The other
 * checks and reports are wc12_decode's, into the one *d_status. */
typedef struct {
  const void *cont;
  uint64_t cont_bytes;
  void *out;
  uint64_t n;
} wc12_decode_item;
WC_API int32_t wc12_decode_batch(const wc12_decode_item *items, uint32_t count, int32_t *d_status,
                                 void *stream);

/* Y = X W^T with W (N x K bf16, row-major) given as a Split12 container, the
 * weights crossing HBM at 12 bits a value ("weight-compression" README:
 * serving with the weights kept in this format).  The weights' planes and X
 * come in by TMA; the weights are expanded tile by tile into the tensor
 * cores' operand layout and multiplied with tcgen05.mma, exact bf16 products
 * accumulated in fp32.
 *   d_w, w_bytes  the container (16-byte aligned, at least 96 bytes, and at
 *                 least up to the end of the low plane an N x K container
 *                 has), n = N * K
 *   N, K          N a multiple of 128, K a multiple of 64
 *   d_x           M x K bf16, row-major, 16-byte aligned; M >= 1 (taken in
 *                 slices of 256 tokens, one launch each)
 *   d_y           M x N fp32, row-major (overwritten)
 *   d_status      device i32 set to 0 by the caller: WC_ERR_CORRUPT for a bad
 *                 container, WC_ERR_TIMEOUT if a bounded wait ran out
 * Returns WC_OK, WC_ERR_INVALID_ARG or WC_ERR_CUDA (also when the driver
 * cannot describe the planes to TMA). */
WC_API int32_t wc12_linear(const void *d_w, uint64_t w_bytes, uint32_t N, uint32_t K,
                           const void *d_x, uint32_t M, float *d_y, int32_t *d_status,
                           void *stream);

/* The serving plan of a container for wc12_linear_planned: the container's
 * exceptions grouped by the tiles the layer works in (128 weight rows x 64
 * values of K), so that each tile finds its exceptions as one range instead
 * of searching the container's per-chunk lists at every call.  Built once
 * per weight matrix; it depends on the container and on N, K only.
 * Layout (little-endian): u32 "W12P", u32 version 1, u32 N, u32 K, u64 ne,
 * u64 buckets = N/128 * K/64; u32 start[buckets + 1] (bucket b * (K/64) + s
 * holds the exceptions of row block b, stage s); then, 16-byte aligned,
 * u32 entry[ne]: column in the stage (bits 0-5), row in the block (bits
 * 6-12), the exception's high byte (bits 16-23), in any order within a
 * bucket. */
WC_API uint64_t wc12_plan_bytes(uint32_t N, uint32_t K, uint64_t ne);

/* Build the plan of container d_w (w_bytes, 16-byte aligned; N x K weights,
 * N a multiple of 128, K of 64; ne its exception count, from
 * wc12_read_header) into d_plan (plan_bytes >= wc12_plan_bytes(N, K, ne),
 * 16-byte aligned).  *d_status (device i32 set to 0 by the caller) receives
 * WC_ERR_CORRUPT if the container's header disagrees with N, K, ne or its
 * exception lists are corrupt; the plan is then marked invalid (its magic
 * is 0) and wc12_linear_planned refuses it.  Four launches on the stream.
 * Returns WC_OK, WC_ERR_INVALID_ARG, WC_ERR_CAPACITY (plan_bytes too small)
 * or WC_ERR_CUDA. */
WC_API int32_t wc12_plan(const void *d_w, uint64_t w_bytes, uint32_t N, uint32_t K, uint64_t ne,
                         void *d_plan, uint64_t plan_bytes, int32_t *d_status, void *stream);

/* wc12_linear with the container's plan (d_plan, plan_bytes; built by
 * wc12_plan for this container and N x K): the same result, without the
 * per-call search for each tile's exceptions.  A plan whose header does not
 * match the container (N, K, ne) is reported as WC_ERR_CORRUPT, as are
 * start offsets out of order.  Returns WC_OK, WC_ERR_INVALID_ARG (also for
 * a null plan or plan_bytes below its header and starts) or WC_ERR_CUDA. */
WC_API int32_t wc12_linear_planned(const void *d_w, uint64_t w_bytes, const void *d_plan,
                                   uint64_t plan_bytes, uint32_t N, uint32_t K, const void *d_x,
                                   uint32_t M, float *d_y, int32_t *d_status, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* WC_SPLIT12_H */
