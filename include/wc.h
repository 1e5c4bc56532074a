/*
 * wc.h -- C ABI of the B200 (sm_100a) exponent-plane rANS weight codec.
 *
 * Lossless compression of bf16 / fp32 / fp16 / fp8 (e4m3, e5m2) weight tensors.
 * Each float is split into planes; the skewed exponent plane is entropy-coded
 * with a static, 32-lane interleaved rANS coder, chunk by chunk; the sign and
 * mantissa bits are stored raw.  Decoding re-merges the planes into the
 * original bits.  The method follows:
 *   - "PTWM" (PyPI README), "How it works": 1. Bit reorder (the exponent
 *     moves to the top, the sign is tucked under it) and 2. Byte / nibble
 *     split (a bf16 value becomes two byte planes, the high one the
 *     exponent); the exponent plane holds ~20 distinct values, the mantissa
 *     planes look random;
 *   - "SMEF -- blog companion code", file table: pass3_streams.py splits
 *     sign / exponent / mantissa streams, pass4_rans.py is the rANS coder;
 *   - "PTWM", Configuration table: compression_threshold (store raw when
 *     coding does not pay) and is_streaming / streaming_chunk (independently
 *     decodable chunks);
 *   - "seedpack 0.2.0 -> 0.2.2", README: a container of chunks plus an index,
 *     with random access.
 *
 * Container (every field little-endian, sections 16-byte aligned, pad bytes
 * zero):  "WCZ1", u16 version 1, u8 dtype, u8 lanes (32), u64 n,
 * u32 chunk symbols (65536), u32 nc, u16 table bits (12), u16 0, u32 0,
 * u64 off_raw, u64 off_exp, u64 exp_bytes, u64 total_bytes (64 bytes), then
 * u16 freq[256], u64 chunk_off[nc+1], u32 chunk_len[nc], the raw planes
 * (bf16: n sign+mantissa bytes; fp32: ceil(n/8) sign-bit bytes, 3n mantissa
 * bytes; fp16: n low bytes; fp8: ceil(n/2) bytes of low nibbles) and
 * the exponent chunks (bf16 / fp32: the exponent byte; fp16: the reordered
 * high byte; fp8 e4m3: the exponent nibble; fp8 e5m2: the top four exponent
 * bits).  Values are passed as raw bits
 * (bf16 / fp16 2 bytes, fp32 4, fp8 1).  A coded chunk is 32 final u32 states then
 * w u16 renormalisation words (128 + 2w bytes); a chunk whose coded form is
 * not smaller than its nsym exponent bytes is stored raw.  The format is
 * fully determined by the input bits: one input has exactly one container.
 *
 * Conventions for every call below:
 *   - Pointers named d_* are device pointers on the current CUDA device;
 *     h_* are host pointers.  The caller owns every buffer.  The library
 *     allocates no memory and never synchronises the device: all work is
 *     queued on `stream` (a cudaStream_t / CUstream handle; NULL is the
 *     legacy default stream) and the call returns before it runs.  It holds
 *     two arrays in device memory of its own, loaded with it on every GPU:
 *     wc_encode_noalloc's scratch (below) and 16 KiB of counters through
 *     which a decode launch's blocks share out its work (4096 slots taken in
 *     turn, each zeroed on the launch's stream first, so that up to 4096
 *     decode launches may overlap on different streams).
 *   - Tensor and container buffers must be 16-byte aligned, scratch 256-byte
 *     aligned.  Values are passed as raw bits (bf16 = 2 bytes, fp32 = 4).
 *   - Argument, alignment and capacity errors are returned synchronously and
 *     queue no work.  Corrupt containers are found on the device: the decode
 *     calls clear *d_status (an int32 in device memory) in stream order and a
 *     kernel stores a non-zero wc_status code there when it rejects a
 *     container; read it after the stream has finished.  A decoder never
 *     writes outside [d_out, d_out + out_cap) and never reads outside
 *     [d_cont, d_cont + cont_bytes).
 *   - WC_ERR_CUDA means a kernel launch failed; cudaGetLastError() in the
 *     library's runtime was consumed and its text is available through
 *     wc_last_error().
 */
#ifndef WC_H
#define WC_H

#include <stdint.h>

#if defined(__GNUC__)
#define WC_API __attribute__((visibility("default")))
#else
#define WC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WC_OK = 0,
    WC_ERR_INVALID_ARG = 1,
    WC_ERR_CAPACITY = 2,
    WC_ERR_CUDA = 3,
    WC_ERR_CORRUPT = 4,
    WC_ERR_UNSUPPORTED = 5,
    WC_ERR_TIMEOUT = 6      /* a kernel's bounded wait ran out (device status) */
} wc_status;

/* WC_FP16: after the reorder S E M -> E S M an fp16 value is cut into its
 * two bytes like a bf16 one and the high byte is coded ("PTWM", How it works
 * 1-2); for fp16 that byte holds the 5 exponent bits, the sign and the top 2
 * mantissa bits, and the raw byte the other 8. */
/* WC_FP8E4M3: the reorder puts the 4 exponent bits in the high nibble and the
 * value is cut into its two nibbles, the exponent nibbles being the coded
 * stream ("PTWM", How it works 1-2); the low nibbles (sign above 3 mantissa
 * bits) are stored raw, two per byte, even value low. */
/* WC_FP8E5M2: the same reorder puts the 5 exponent bits on top; the value is
 * cut into nibbles as for e4m3, so the coded stream is the high nibble
 * (exponent bits 4..1) and the raw nibble holds exponent bit 0, the sign and
 * the 2 mantissa bits ("PTWM", Supported dtypes: float8_e5m2 takes the same
 * bit reorder and 2-plane nibble split as float8_e4m3). */
typedef enum { WC_BF16 = 1, WC_FP32 = 2, WC_FP16 = 3, WC_FP8E4M3 = 4, WC_FP8E5M2 = 5 } wc_dtype;

/* Worst-case container size in bytes for n values of dtype: every chunk
 * stored raw ("PTWM" Configuration table, compression_threshold: the coded
 * form is only kept when it is smaller).  0 for an unknown dtype. */
WC_API uint64_t wc_encode_bound(uint64_t n, int32_t dtype);

/* Device scratch bytes wc_encode needs for n values (about 66 KiB per
 * 65,536-value chunk plus a 6.25 KiB table area).  0 for an unknown dtype. */
WC_API uint64_t wc_scratch_bytes(uint64_t n, int32_t dtype);

/* Encode n values at d_in into a container at d_out.
 *   d_in        n raw values (bf16 bits or fp32 bits), 16-byte aligned.
 *   out_cap     bytes available at d_out; must be >= wc_encode_bound(n).
 *   d_scratch   >= wc_scratch_bytes(n) bytes, 256-byte aligned; its content
 *               on entry does not matter and is garbage on return.
 *   d_out_size  device u64 receiving the container size in bytes.
 * Steps ("PTWM" How it works 1-2; "SMEF" pass 3 and pass 4): plane split and
 * per-tensor exponent histogram, the 12-bit table (sum 4096, every present
 * exponent >= 1), 32-lane rANS per 65,536-value chunk with the raw fallback,
 * exclusive scan of the chunk sizes into the offset table, and compaction.
 * Returns WC_OK, WC_ERR_INVALID_ARG, WC_ERR_CAPACITY or WC_ERR_CUDA. */
WC_API int32_t wc_encode(const void *d_in, uint64_t n, int32_t dtype, void *d_out,
                  uint64_t out_cap, void *d_scratch, uint64_t scratch_cap,
                  uint64_t *d_out_size, void *stream);

/* Decode a whole container into d_out (n values of the container's dtype,
 * 16-byte aligned, out_cap bytes).  The header is read on the device, so the
 * host needs no copy of it; a container whose n values do not fit in out_cap
 * is rejected on the device with WC_ERR_CAPACITY in *d_status.  Decoding
 * inverts each chunk's rANS stream and re-merges the planes into the
 * original bits ("PTWM" How it works; "SMEF" pass 3 merge_streams).
 * Returns WC_OK, WC_ERR_INVALID_ARG or WC_ERR_CUDA; container problems go to
 * *d_status (WC_ERR_CORRUPT / WC_ERR_CAPACITY). */
WC_API int32_t wc_decode(const void *d_cont, uint64_t cont_bytes, void *d_out,
                  uint64_t out_cap, int32_t *d_status, void *stream);

/* Random access: decode only chunk k, i.e. values [65536 k, min(n, 65536 (k+1)))
 * into d_out[0 ...] ("PTWM" Random access; "seedpack" README, chunks plus
 * index).  k >= nc is reported as WC_ERR_INVALID_ARG in *d_status. */
WC_API int32_t wc_decode_chunk(const void *d_cont, uint64_t cont_bytes, uint64_t k,
                        void *d_out, uint64_t out_cap, int32_t *d_status,
                        void *stream);

/* Parse and check the fixed header at h_cont (host memory, >= 64 bytes;
 * the offset table is checked too when it is present in the bytes given).
 * Returns WC_OK or WC_ERR_CORRUPT / WC_ERR_INVALID_ARG. */
WC_API int32_t wc_read_header(const void *h_cont, uint64_t bytes, uint64_t *n,
                       int32_t *dtype, uint64_t *nchunks);

/* Batched calls: many tensors in one launch per kernel (a whole model's
 * weight set in a handful of launches).  The item arrays are host memory;
 * the pointers inside are device pointers with the meaning and alignment of
 * the single-tensor calls.  Every item is validated before anything is
 * queued; on an error no work is queued.  Items may use any sizes, including
 * n = 0. */
typedef struct {
    const void *in;       /* n values, 16-byte aligned                   */
    uint64_t n;
    int32_t dtype;        /* a wc_dtype                                  */
    int32_t reserved;     /* must be 0                                   */
    void *out;            /* container, out_cap >= wc_encode_bound(n)    */
    uint64_t out_cap;
    void *scratch;        /* >= wc_scratch_bytes(n), 256-byte aligned    */
    uint64_t scratch_cap;
    uint64_t *out_size;   /* device u64                                  */
} wc_encode_item;

typedef struct {
    const void *cont;     /* container, 16-byte aligned                  */
    uint64_t cont_bytes;
    void *out;            /* decoded values, 16-byte aligned             */
    uint64_t out_cap;
} wc_decode_item;

WC_API int32_t wc_encode_batch(const wc_encode_item *h_items, uint32_t count,
                        void *stream);
WC_API int32_t wc_decode_batch(const wc_decode_item *h_items, uint32_t count,
                        int32_t *d_status, void *stream);

/* Encoding with no scratch buffer from the caller.  (The pages have no
 * counterpart; this exists for callers of the library.)
 *
 * For callers that cannot allocate device memory where they encode: a runtime
 * that owns all device memory through a fixed, pre-planned arena and forbids
 * allocations outside it, a plug-in that another framework calls with only
 * its input and output buffers, or a latency-critical path that cannot afford
 * an allocator's implicit synchronisation.  Arguments and results are those of
 * wc_encode without d_scratch / scratch_cap; the scratch is a device array of
 * WC_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads it,
 * from load until the process exits.  That limits n to values whose
 * wc_scratch_bytes(n) fits: 16,252,928 values (248 chunks) for either dtype;
 * larger inputs are rejected with WC_ERR_CAPACITY before any work is queued,
 * and a failed device-address lookup returns WC_ERR_CUDA.
 *
 * The first call on a device looks up the array's device address with that
 * device current (a host-side lookup, cached per device and CUDA context: a
 * call after the context was destroyed and created again, e.g. by
 * cudaDeviceReset, looks it up again); make that first call before capturing
 * any stream on that device.  All calls on a GPU share the
 * one array: calls whose work overlaps on the GPU (for example on two streams
 * without ordering between them) race and corrupt each other's output; calls
 * queued on one stream, or otherwise ordered, do not.  The array's contents
 * between calls do not matter: each call clears the parts that must start at
 * zero. */
#define WC_NOALLOC_SCRATCH_BYTES (16u << 20)
WC_API int32_t wc_encode_noalloc(const void *d_in, uint64_t n, int32_t dtype, void *d_out,
                                 uint64_t out_cap, uint64_t *d_out_size, void *stream);

/* Host-resident tensors, encoded and decoded through the device in windows
 * ("seedpack 0.2.0 -> 0.2.2", README: a BF16 model larger than the GPU's
 * memory is handled in groups of tensors of roughly a gigabyte and unpacked
 * on the GPU one tensor after another).
 *
 * The items' buffers (h_*) are host memory; on the device the calls use only
 * the caller's workspace d_work (256-byte aligned, work_cap bytes).  The
 * workspace is cut into slots; consecutive items are grouped into windows
 * that fit one slot (wc_host_plan), and the windows go through a pipeline:
 * host->device copies on stream_in, the batched kernels on stream_compute,
 * device->host copies on stream_out, ordered by events, so that copies in
 * both directions and the kernels of consecutive windows overlap.  Host
 * buffers must be page-locked for the copies to overlap; pageable memory
 * works but serialises them.  The three streams may be one stream (no
 * overlap).  Containers and decoded values are exactly those of
 * wc_encode_batch / wc_decode_batch.
 *
 * Unlike the calls above, these two block: they return after every copy has
 * finished (or at the first error, after the work already queued is done) and
 * synchronise the three streams.  Each call creates and destroys a few CUDA
 * events (and wc_encode_host one more stream, for reading sizes back); no
 * memory is allocated.  Argument, header and capacity checks come
 * first and queue no work.
 *
 * Workspace: 256-byte rounded 4 * count bytes of status words, then the
 * slots.  An item needs wc_host_encode_footprint / wc_host_decode_footprint
 * bytes of a slot (a window adds 256).  Three slots are used when each can
 * hold the largest item, else two, else one; if one slot cannot hold it the
 * call returns WC_ERR_CAPACITY. */
typedef struct {
    const void *h_in;       /* n values (host)                              */
    uint64_t n;
    int32_t dtype;          /* a wc_dtype                                   */
    int32_t reserved;       /* must be 0                                    */
    void *h_out;            /* container (host)                             */
    uint64_t h_out_cap;     /* must be >= wc_encode_bound(n, dtype)         */
    uint64_t *h_out_size;   /* host u64: the container's size               */
} wc_host_encode_item;

typedef struct {
    const void *h_cont;     /* container (host); its header is read here    */
    uint64_t cont_bytes;
    void *h_out;            /* decoded values (host), n * element bytes     */
    uint64_t out_cap;
} wc_host_decode_item;

/* Slot bytes one item needs (0 for an unknown dtype or n > 2^44). */
WC_API uint64_t wc_host_encode_footprint(uint64_t n, int32_t dtype);
WC_API uint64_t wc_host_decode_footprint(uint64_t cont_bytes, uint64_t n, int32_t dtype);

/* The window plan the two calls use (host arithmetic only, no CUDA call):
 * *slots = 3, 2 or 1 -- the most slots of 256-byte rounded (slot_area /
 * slots) bytes that each hold the largest footprint plus 256 -- and greedy
 * windows of consecutive items whose footprints plus 256 stay within
 * min(slot, window_bytes) (window_bytes = 0: the slot), except that an item
 * larger than that gets a window of its own.  Window w holds items
 * [window_end[w-1], window_end[w]) (window_end[-1] = 0); *n_windows <= count
 * and window_end needs room for count entries.  Smaller windows give the
 * pipeline more stages to overlap.  WC_ERR_CAPACITY if no slot count fits,
 * WC_ERR_INVALID_ARG for a null pointer or a zero footprint. */
WC_API int32_t wc_host_plan(const uint64_t *h_footprints, uint32_t count, uint64_t slot_area,
                            uint64_t window_bytes, uint32_t *slots, uint32_t *window_end,
                            uint32_t *n_windows);

WC_API int32_t wc_encode_host(const wc_host_encode_item *h_items, uint32_t count, void *d_work,
                              uint64_t work_cap, uint64_t window_bytes, void *stream_in,
                              void *stream_compute, void *stream_out);

/* *h_status: WC_OK, or the device status of the first window with a
 * rejected container (its outputs are then undefined). */
WC_API int32_t wc_decode_host(const wc_host_decode_item *h_items, uint32_t count, void *d_work,
                              uint64_t work_cap, uint64_t window_bytes, void *stream_in,
                              void *stream_compute, void *stream_out, int32_t *h_status);

/* The byte ranges of a container that wc_decode_chunk reads for chunk k:
 * random access inside a stored tensor ("PTWM", Random access: a reader
 * fetches what one tensor needs without reading the rest) can copy just these
 * to the device and leave the rest of a container-sized buffer unwritten.
 *   h_prefix      host copy of the container's first prefix_bytes bytes; it
 *                 must reach the end of the tables, i.e. the raw-plane offset
 *                 stored at header byte 32 (WC_ERR_CAPACITY otherwise).
 *   k             the chunk (WC_ERR_INVALID_ARG if k >= nchunks).
 *   ranges        host, 8 uint64: up to 4 {offset, bytes} pairs in ascending
 *                 order, written for *count of them: the header and tables
 *                 [0, raw-plane offset), the chunk's raw-plane bytes (two
 *                 ranges for fp32: sign bits and mantissa bytes), and its
 *                 exponent payload rounded up to 16 bytes.
 * The header and chunk k's offset-table entries are checked as wc_read_header
 * and the decoder check them (WC_ERR_CORRUPT).  Host only; no device work. */
WC_API int32_t wc_chunk_ranges(const void *h_prefix, uint64_t prefix_bytes, uint64_t k,
                               uint64_t *ranges, uint32_t *count);

/* CRC-32 of fixed-size blocks of a device buffer, the per-block check that
 * an archive file keeps ("seedpack 0.2.0 -> 0.2.2", README: every chunk of an
 * archive carries a CRC32).  The code is zlib's and IEEE 802.3's CRC-32
 * (generator 0x04C11DB7, bits least significant first, register preset to
 * all ones, result complemented; "123456789" gives 0xCBF43926).
 *   d_buf        device, 16-byte aligned, `bytes` bytes (read only).  bytes
 *                = 0 is allowed and queues nothing.
 *   block_bytes  the block size: a multiple of 8192, at most 2^30.  Block i
 *                is [i * block_bytes, min((i + 1) * block_bytes, bytes)).
 *   d_crc        device, ceil(bytes / block_bytes) uint32, written in block
 *                order.
 * Queued on `stream`; returns WC_OK, WC_ERR_INVALID_ARG (null or misaligned
 * pointer, bad block size) or WC_ERR_CUDA. */
WC_API int32_t wc_crc32_blocks(const void *d_buf, uint64_t bytes, uint64_t block_bytes,
                               uint32_t *d_crc, void *stream);

/* Human-readable name of a wc_status code (static storage). */
WC_API const char *wc_status_string(int32_t status);

/* Text of the last CUDA error the library saw on this thread ("" if none). */
WC_API const char *wc_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* WC_H */
