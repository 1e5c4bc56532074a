/*
 * wc_oracle.h -- declarations of the CPU oracle for the exponent-plane rANS
 * weight container.
 *
 * TEST INFRASTRUCTURE ONLY.  This header and wc_oracle.c are the slow, plain,
 * scalar reference that the CUDA library is checked against.  Only the test
 * suite, the smoke check and the CPU-baseline leg of the benchmark may load
 * it.  It shares no code, header, table or constant with the CUDA library:
 * every constant below is restated here on purpose.
 *
 * All functions return 0 on success and one of the OR_ERR_* codes otherwise.
 */
#ifndef WC_ORACLE_H
#define WC_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    OR_OK = 0,
    OR_ERR_INVALID_ARG = 1,
    OR_ERR_CAPACITY = 2,
    OR_ERR_CORRUPT = 4
};

/* 5: fp8 e5m2; 6: bf16 split into its bytes without the reorder (the high
 * byte S E7..E1 coded, the low byte E0 M7 raw): the Split12 split, kept as a
 * comparison against the reorder. */
enum { OR_BF16 = 1, OR_FP32 = 2, OR_FP16 = 3, OR_FP8E4M3 = 4, OR_FP8E5M2 = 5,
       OR_BF16_HIGHBYTE = 6 };

/* Worst-case container size (every chunk stored raw). */
uint64_t oracle_encode_bound(uint64_t n, int dtype);

/* Plane split (PTWM README, "How it works" 1-2; SMEF README, pass 3). */
void oracle_split_bf16(const uint16_t *in, uint64_t n, uint8_t *exp_plane,
                       uint8_t *sm_plane);
void oracle_split_fp32(const uint32_t *in, uint64_t n, uint8_t *exp_plane,
                       uint8_t *sign_bits, uint8_t *mant3);
void oracle_split_fp16(const uint16_t *in, uint64_t n, uint8_t *hi_plane,
                       uint8_t *lo_plane);
void oracle_split_fp8e4m3(const uint8_t *in, uint64_t n, uint8_t *exp_plane,
                          uint8_t *nibble_plane);
void oracle_split_fp8e5m2(const uint8_t *in, uint64_t n, uint8_t *hi_nibbles,
                          uint8_t *nibble_plane);
void oracle_split_bf16_highbyte(const uint16_t *in, uint64_t n, uint8_t *hi_plane,
                                uint8_t *lo_plane);

/* 256-bin count of an exponent plane. */
void oracle_histogram(const uint8_t *exp_plane, uint64_t n, uint64_t counts[256]);

/* counts -> 12-bit table (sum 4096, every present symbol >= 1). */
int oracle_normalize(const uint64_t counts[256], uint16_t freq[256]);

/* Static rANS core for one chunk, with a lane count parameter (1 or 32 are
 * used by the tests).  words must hold nsym entries.  No raw fallback here. */
int oracle_rans_encode(const uint8_t *sym, uint32_t nsym, const uint16_t freq[256],
                       uint32_t lanes, uint32_t *states_out, uint16_t *words_out,
                       uint32_t *nwords_out);
int oracle_rans_decode(const uint32_t *states_in, const uint16_t *words,
                       uint32_t nwords, uint32_t nsym, const uint16_t freq[256],
                       uint32_t lanes, uint8_t *sym_out);

/* Whole container. */
int oracle_encode(const void *in, uint64_t n, int dtype, uint8_t *out,
                  uint64_t out_cap, uint64_t *out_size);
int oracle_decode(const uint8_t *cont, uint64_t cont_bytes, void *out,
                  uint64_t out_cap);
int oracle_decode_chunk(const uint8_t *cont, uint64_t cont_bytes, uint64_t k,
                        void *out, uint64_t out_cap);
int oracle_read_header(const uint8_t *cont, uint64_t cont_bytes, uint64_t *n,
                       int *dtype, uint64_t *nchunks);

/* Diagnostic: for one chunk coded with the given table, the exact rANS
 * accounting terms (see wc_oracle.c). */
int oracle_chunk_accounting(const uint8_t *sym, uint32_t nsym,
                            const uint16_t freq[256], double *coded_bits,
                            double *ideal_bits, double *slack_bound);

/* CRC-32 of a byte string as zlib and IEEE 802.3 define it: generator
 * x^32 + x^26 + x^23 + x^22 + x^16 + x^12 + x^11 + x^10 + x^8 + x^7 + x^5 +
 * x^4 + x^2 + x + 1, bits taken least significant first, register preset to
 * all ones and complemented at the end ("seedpack 0.2.0 -> 0.2.2", README:
 * every chunk of an archive carries a CRC32). */
uint32_t oracle_crc32(const uint8_t *data, uint64_t bytes);
/* The CRC-32 of each block [i*block_bytes, min((i+1)*block_bytes, bytes)),
 * i < ceil(bytes / block_bytes), into crc[i]. */
int oracle_crc32_blocks(const uint8_t *data, uint64_t bytes, uint64_t block_bytes,
                        uint32_t *crc);

#ifdef __cplusplus
}
#endif
#endif
