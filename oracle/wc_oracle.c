/*
 * wc_oracle.c -- plain, scalar CPU oracle of the exponent-plane rANS weight
 * container.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * statement of what the CUDA library must compute, byte for byte.  Only the
 * test suite, the smoke check and the CPU-baseline leg of the benchmark may
 * load it; the library itself never does.  It shares no code, header, table or
 * constant with the CUDA sources.  It is written for reading, not for speed:
 * one value at a time, one symbol at a time, plain u32/u64 arithmetic with
 * hardware division, no blocking, no fusion.
 *
 * What the method is, and where each step comes from:
 *
 *  - Plane split.  A float is split into byte/bit planes so that the skewed
 *    exponent is separated from the mantissa, whose bits look random ("SMEF -- blog
 *    companion code", file table, pass3_streams.py, and "Reading order" item 1;
 *    "PTWM", "How it works" 1. Bit reorder and 2. Byte / nibble split).  For
 *    bf16 the exponent byte is the high byte after the reorder
 *    [S E M] -> [E S M], and the low byte holds the sign above the 7 mantissa
 *    bits.  For fp16 the same reorder and 2-plane byte split give a coded
 *    high byte of 5 exponent bits, the sign and the top 2 mantissa bits, and
 *    a raw low byte of the other 8 mantissa bits ("PTWM", "How it works" 2:
 *    16-bit floats are cut into their two bytes, the high byte being the
 *    exponent-bearing one).
 *    For fp8 e4m3 the reorder S E M -> E S M puts the 4 exponent bits in the
 *    high nibble and a nibble split separates them ("PTWM", "How it works"
 *    1-2: 8-bit floats are cut into two nibbles, the exponent nibbles forming
 *    a stream of their own): the coded symbol is the exponent nibble, and the low nibbles
 *    (sign above 3 mantissa bits) are stored raw, two per byte.
 *    For fp32 the container keeps three streams: sign bits, the 8-bit
 *    exponent, and the 23-bit mantissa stored as 3 little-endian bytes.
 *
 *  - Entropy coder.  Only the exponent plane is coded, with static rANS ("SMEF
 *    -- blog companion code", pass4_rans.py; "PTWM", "How it works" 2, where
 *    the exponent plane carries ~20 distinct values and ~2.6 bits/byte).  The
 *    container fixes: a per-tensor 12-bit frequency table (sum 4096), 32-bit
 *    states kept in [2^16, 2^32), 16-bit renormalisation words, 32 interleaved
 *    lanes (symbol i in lane i mod 32), 65,536-symbol chunks.
 *
 *  - Raw fallback.  A chunk whose coded form is not smaller than its raw
 *    exponent bytes is stored raw ("PTWM", Configuration table,
 *    compression_threshold: store raw when compression does not pay).
 *
 *  - Random access.  Chunks are independently decodable and located through a
 *    per-chunk offset table ("PTWM", Configuration table, is_streaming /
 *    streaming_chunk; "seedpack 0.2.0 -> 0.2.2", README, chunks plus an index
 *    for random access).
 *
 * The pages give no table-normalisation rule, no lane layout, no word order
 * and no byte layout.  The readings chosen for those are stated at each
 * function below; they define the container.
 *
 * Container layout (all fields little-endian, sections 16-byte aligned,
 * padding bytes zero):
 *   0  "WCZ1"            4  u16 version = 1    6  u8 dtype (1 bf16, 2 fp32, 3 fp16,
 *                                              4 fp8 e4m3)
 *   7  u8 lanes = 32     8  u64 n              16 u32 chunk symbols = 65536
 *   20 u32 nc            24 u16 prob bits = 12 26 u16 0      28 u32 0
 *   32 u64 off_raw       40 u64 off_exp        48 u64 exp_bytes
 *   56 u64 total_bytes   64 u16 freq[256]      576 u64 chunk_off[nc + 1]
 *   then u32 chunk_len[nc]; pad; raw section; pad; exponent section.
 *   bf16 raw section: n sign+mantissa bytes; fp16: n low bytes; fp8 e4m3:
 *   ceil(n/2) bytes of low nibbles (value 2j in the low half of byte j).
 *   fp32 raw section: ceil(n/8) sign bytes (value 8j+b is bit b of byte j),
 *   pad, then 3n mantissa bytes.
 *   Exponent section: chunk k at off_exp + chunk_off[k], chunk_len[k] bytes,
 *   zero-padded to a multiple of 16; chunk_off[k+1] = chunk_off[k] +
 *   round16(chunk_len[k]).  A coded chunk is [32 final states, u32][w words,
 *   u16] (length 128 + 2w); a raw chunk is its nsym exponent bytes.
 */
#include "wc_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define OR_CHUNK_SYMBOLS 65536u
#define OR_LANES 32u
#define OR_PROB_BITS 12u
#define OR_PROB_SCALE 4096u      /* 2^12 */
#define OR_STATE_LOW 65536u      /* L = 2^16, lower end of the state interval */
#define OR_HEADER_BYTES 64u
#define OR_FREQ_OFFSET 64u
#define OR_CHUNK_OFF_OFFSET 576u /* 64 + 2*256 */

/* ------------------------------------------------------------------ */
/* Little-endian byte access, one byte at a time.                      */
/* ------------------------------------------------------------------ */
static void put_u16(uint8_t *p, uint16_t v) {
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)(v >> 8);
}
static void put_u32(uint8_t *p, uint32_t v) {
    for (int b = 0; b < 4; b++) p[b] = (uint8_t)(v >> (8 * b));
}
static void put_u64(uint8_t *p, uint64_t v) {
    for (int b = 0; b < 8; b++) p[b] = (uint8_t)(v >> (8 * b));
}
static uint16_t get_u16(const uint8_t *p) {
    return (uint16_t)(p[0] | (p[1] << 8));
}
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int b = 3; b >= 0; b--) v = (v << 8) | p[b];
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int b = 7; b >= 0; b--) v = (v << 8) | p[b];
    return v;
}

static uint64_t round_up16(uint64_t v) { return (v + 15u) / 16u * 16u; }

/* ------------------------------------------------------------------ */
/* Section layout, a pure function of n and dtype.                     */
/* ------------------------------------------------------------------ */
typedef struct {
    uint64_t n, nc;
    uint64_t off_chunk_off, off_chunk_len;
    uint64_t off_raw, off_sign, off_mant, off_exp;
} or_layout;

static void or_make_layout(uint64_t n, int dtype, or_layout *lay) {
    lay->n = n;
    lay->nc = (n + OR_CHUNK_SYMBOLS - 1) / OR_CHUNK_SYMBOLS;
    lay->off_chunk_off = OR_CHUNK_OFF_OFFSET;
    lay->off_chunk_len = lay->off_chunk_off + 8 * (lay->nc + 1);
    lay->off_raw = round_up16(lay->off_chunk_len + 4 * lay->nc);
    if (dtype == OR_BF16 || dtype == OR_FP16 || dtype == OR_BF16_HIGHBYTE) {
        lay->off_sign = 0;
        lay->off_mant = 0;
        lay->off_exp = round_up16(lay->off_raw + n);
    } else if (dtype == OR_FP8E4M3 || dtype == OR_FP8E5M2) {
        lay->off_sign = 0;
        lay->off_mant = 0;
        lay->off_exp = round_up16(lay->off_raw + (n + 1) / 2);
    } else {
        lay->off_sign = lay->off_raw;
        lay->off_mant = round_up16(lay->off_raw + (n + 7) / 8);
        lay->off_exp = round_up16(lay->off_mant + 3 * n);
    }
}

static uint32_t or_chunk_nsym(uint64_t n, uint64_t k) {
    uint64_t first = k * OR_CHUNK_SYMBOLS;
    uint64_t left = n - first;
    return (uint32_t)(left < OR_CHUNK_SYMBOLS ? left : OR_CHUNK_SYMBOLS);
}

static int or_dtype_ok(int dtype) {
    return dtype == OR_BF16 || dtype == OR_FP32 || dtype == OR_FP16 || dtype == OR_FP8E4M3 ||
           dtype == OR_FP8E5M2 || dtype == OR_BF16_HIGHBYTE;
}

/* Bytes per value of a dtype. */
static uint64_t or_elem(int dtype) {
    return dtype == OR_FP32 ? 4 : (dtype == OR_FP8E4M3 || dtype == OR_FP8E5M2 ? 1 : 2);
}

uint64_t oracle_encode_bound(uint64_t n, int dtype) {
    or_layout lay;
    if (!or_dtype_ok(dtype)) return 0;
    or_make_layout(n, dtype, &lay);
    uint64_t exp_bytes = 0;
    for (uint64_t k = 0; k < lay.nc; k++) exp_bytes += round_up16(or_chunk_nsym(n, k));
    return lay.off_exp + exp_bytes;
}

/* ------------------------------------------------------------------ */
/* Plane split ("PTWM", How it works 1-2; "SMEF", pass3_streams.py).   */
/* ------------------------------------------------------------------ */

/* bf16 bits b = [S:1][E:8][M:7].  After the reorder [E S M] the high byte is
 * E and the low byte is S above M: sm = S<<7 | M. */
void oracle_split_bf16(const uint16_t *in, uint64_t n, uint8_t *exp_plane,
                       uint8_t *sm_plane) {
    for (uint64_t i = 0; i < n; i++) {
        uint16_t b = in[i];
        uint8_t sign = (uint8_t)((b >> 15) & 1u);
        uint8_t expo = (uint8_t)((b >> 7) & 0xFFu);
        uint8_t mant = (uint8_t)(b & 0x7Fu);
        exp_plane[i] = expo;
        sm_plane[i] = (uint8_t)((sign << 7) | mant);
    }
}

/* fp32 bits u = [S:1][E:8][M:23]: sign bits packed least-significant bit
 * first (value 8j+b -> bit b of byte j), exponent byte, mantissa as 3
 * little-endian bytes.  sign_bits must be zeroed by the caller. */
void oracle_split_fp32(const uint32_t *in, uint64_t n, uint8_t *exp_plane,
                       uint8_t *sign_bits, uint8_t *mant3) {
    for (uint64_t i = 0; i < n; i++) {
        uint32_t u = in[i];
        uint32_t sign = u >> 31;
        uint32_t expo = (u >> 23) & 0xFFu;
        uint32_t mant = u & 0x7FFFFFu;
        exp_plane[i] = (uint8_t)expo;
        if (sign) sign_bits[i / 8] = (uint8_t)(sign_bits[i / 8] | (1u << (i % 8)));
        mant3[3 * i + 0] = (uint8_t)(mant & 0xFFu);
        mant3[3 * i + 1] = (uint8_t)((mant >> 8) & 0xFFu);
        mant3[3 * i + 2] = (uint8_t)((mant >> 16) & 0xFFu);
    }
}

/* fp16 bits b = [S:1][E:5][M:10].  The reorder puts E on top with S below
 * it: r = E<<11 | S<<10 | M; the byte split gives the high byte r >> 8
 * (E, S and the top two mantissa bits; the coded plane) and the low byte
 * r & 0xFF (the low eight mantissa bits; stored raw). */
void oracle_split_fp16(const uint16_t *in, uint64_t n, uint8_t *hi_plane,
                       uint8_t *lo_plane) {
    for (uint64_t i = 0; i < n; i++) {
        uint16_t b = in[i];
        uint16_t sign = (uint16_t)((b >> 15) & 1u);
        uint16_t expo = (uint16_t)((b >> 10) & 0x1Fu);
        uint16_t mant = (uint16_t)(b & 0x3FFu);
        uint16_t r = (uint16_t)((expo << 11) | (sign << 10) | mant);
        hi_plane[i] = (uint8_t)(r >> 8);
        lo_plane[i] = (uint8_t)(r & 0xFFu);
    }
}

/* fp8 e4m3 bits b = [S:1][E:4][M:3].  The reorder gives E<<4 | S<<3 | M; the
 * nibble split gives the exponent nibble E (coded) and the low nibble
 * S<<3 | M (raw), packed two per byte: value i goes to byte i/2, in the low
 * nibble when i is even.  nibble_plane must be zeroed by the caller. */
void oracle_split_fp8e4m3(const uint8_t *in, uint64_t n, uint8_t *exp_plane,
                          uint8_t *nibble_plane) {
    for (uint64_t i = 0; i < n; i++) {
        uint8_t b = in[i];
        uint8_t sign = (uint8_t)((b >> 7) & 1u);
        uint8_t expo = (uint8_t)((b >> 3) & 0xFu);
        uint8_t mant = (uint8_t)(b & 7u);
        uint8_t r = (uint8_t)((expo << 4) | (sign << 3) | mant);
        exp_plane[i] = (uint8_t)(r >> 4);
        uint8_t lo = (uint8_t)(r & 0xFu);
        nibble_plane[i / 2] = (uint8_t)(nibble_plane[i / 2] | (i % 2 ? lo << 4 : lo));
    }
}

/* fp8 e5m2 bits b = [S:1][E:5][M:2].  The same reorder gives E<<3 | S<<2 | M:
 * the five exponent bits on top.  The nibble split then takes the high nibble
 * (the top four exponent bits; coded) and the low nibble (lowest exponent bit,
 * sign, two mantissa bits; raw), packed as for e4m3. */
void oracle_split_fp8e5m2(const uint8_t *in, uint64_t n, uint8_t *hi_nibbles,
                          uint8_t *nibble_plane) {
    for (uint64_t i = 0; i < n; i++) {
        uint8_t b = in[i];
        uint8_t sign = (uint8_t)((b >> 7) & 1u);
        uint8_t expo = (uint8_t)((b >> 2) & 0x1Fu);
        uint8_t mant = (uint8_t)(b & 3u);
        uint8_t r = (uint8_t)((expo << 3) | (sign << 2) | mant);
        hi_nibbles[i] = (uint8_t)(r >> 4);
        uint8_t lo = (uint8_t)(r & 0xFu);
        nibble_plane[i / 2] = (uint8_t)(nibble_plane[i / 2] | (i % 2 ? lo << 4 : lo));
    }
}

/* bf16 bits cut into bytes as they are, no reorder: the high byte (sign and
 * the top seven exponent bits) is coded, the low byte (lowest exponent bit
 * and the mantissa) is stored raw ("weight-compression" README: Split12
 * splits bf16 into bytes, rebuilds the high byte from a codebook and keeps the
 * low byte raw). */
void oracle_split_bf16_highbyte(const uint16_t *in, uint64_t n, uint8_t *hi_plane,
                                uint8_t *lo_plane) {
    for (uint64_t i = 0; i < n; i++) {
        hi_plane[i] = (uint8_t)(in[i] >> 8);
        lo_plane[i] = (uint8_t)(in[i] & 0xFFu);
    }
}

void oracle_histogram(const uint8_t *exp_plane, uint64_t n, uint64_t counts[256]) {
    for (int s = 0; s < 256; s++) counts[s] = 0;
    for (uint64_t i = 0; i < n; i++) counts[exp_plane[i]] += 1;
}

/* ------------------------------------------------------------------ */
/* Table normalisation.  The pages fix no rule; the container's rule:  */
/*   f_s = 0 if c_s = 0, else max(1, floor(c_s * 4096 / n));           */
/*   d = 4096 - sum f;                                                 */
/*   d > 0: the symbol with the largest count (lowest symbol on ties)  */
/*          takes all of d;                                            */
/*   d < 0: -d times, the symbol with the largest f among f > 1        */
/*          (lowest symbol on ties) gives up 1.                        */
/* n = 0 gives the all-zero table.  A single present symbol gets 4096. */
/* ------------------------------------------------------------------ */
int oracle_normalize(const uint64_t counts[256], uint16_t freq[256]) {
    uint64_t n = 0;
    for (int s = 0; s < 256; s++) n += counts[s];
    for (int s = 0; s < 256; s++) freq[s] = 0;
    if (n == 0) return OR_OK;

    uint32_t f[256];
    int64_t total = 0;
    for (int s = 0; s < 256; s++) {
        if (counts[s] == 0) {
            f[s] = 0;
        } else {
            /* counts[s] * 4096 < 2^64 for any n < 2^52 */
            uint64_t scaled = counts[s] * (uint64_t)OR_PROB_SCALE / n;
            f[s] = scaled < 1 ? 1u : (uint32_t)scaled;
        }
        total += f[s];
    }
    int64_t d = (int64_t)OR_PROB_SCALE - total;
    if (d > 0) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (counts[s] > 0 && (best < 0 || counts[s] > counts[best])) best = s;
        f[best] += (uint32_t)d;
    }
    while (d < 0) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (f[s] > 1 && (best < 0 || f[s] > f[best])) best = s;
        if (best < 0) return OR_ERR_INVALID_ARG; /* cannot happen: <= 256 symbols */
        f[best] -= 1;
        d += 1;
    }
    for (int s = 0; s < 256; s++) freq[s] = (uint16_t)f[s];
    return OR_OK;
}

/* cum_s = sum of f_t over t < s; slot j in [cum_s, cum_s + f_s) belongs to s. */
static void or_cumulative(const uint16_t freq[256], uint32_t cum[256]) {
    uint32_t c = 0;
    for (int s = 0; s < 256; s++) {
        cum[s] = c;
        c += freq[s];
    }
}

/* ------------------------------------------------------------------ */
/* rANS core for one chunk.                                            */
/*                                                                     */
/* Encoding one symbol s (frequency f, cumulative c) into state x:     */
/*   if (x >> 20) >= f: emit the word x & 0xFFFF and set x = x >> 16;  */
/*   x = (x / f) * 4096 + (x % f) + c.                                 */
/* (x >> 20 >= f is x >= f * 2^20 = ((L >> 12) << 16) * f, written so  */
/*  that f = 4096 does not overflow 32 bits.)  Decoding is the inverse: */
/*   slot = x & 4095; s = symbol owning slot;                          */
/*   x = f * (x >> 12) + slot - c; if x < 2^16: x = x << 16 | word.    */
/*                                                                     */
/* Interleaving: symbol i is coded in lane i mod lanes at step         */
/* t = i / lanes.  The decoder runs t = 0, 1, ... and, within a step,  */
/* lanes in ascending order, reading the next word of one shared       */
/* stream whenever a lane's state falls below 2^16.  The encoder runs  */
/* t = last, ..., 0 and fills the stream from its end: the k lanes     */
/* that emit at step t write one block that ends at the current tail,  */
/* the r-th emitting lane (ascending lane order) at tail - k + r.      */
/* Every lane starts at x = 2^16, so a correct decode ends with every  */
/* lane back at 2^16 and every word consumed.                          */
/* ------------------------------------------------------------------ */
int oracle_rans_encode(const uint8_t *sym, uint32_t nsym, const uint16_t freq[256],
                       uint32_t lanes, uint32_t *states_out, uint16_t *words_out,
                       uint32_t *nwords_out) {
    if (lanes == 0 || lanes > 1024) return OR_ERR_INVALID_ARG;
    uint32_t cum[256];
    or_cumulative(freq, cum);
    for (uint32_t i = 0; i < nsym; i++)
        if (freq[sym[i]] == 0) return OR_ERR_INVALID_ARG;

    uint32_t *x = (uint32_t *)malloc(sizeof(uint32_t) * lanes);
    int *emits = (int *)malloc(sizeof(int) * lanes);
    uint16_t *rev = (uint16_t *)malloc(sizeof(uint16_t) * (nsym + 1));
    if (!x || !emits || !rev) {
        free(x); free(emits); free(rev);
        return OR_ERR_INVALID_ARG;
    }
    for (uint32_t l = 0; l < lanes; l++) x[l] = OR_STATE_LOW;

    /* The stream is built from its end: rev[tail .. nsym) holds it. */
    uint32_t tail = nsym;
    uint32_t steps = (nsym + lanes - 1) / lanes;
    for (uint32_t tt = steps; tt-- > 0;) {
        /* which lanes emit at this step */
        uint32_t k = 0;
        for (uint32_t l = 0; l < lanes; l++) {
            uint64_t i = (uint64_t)tt * lanes + l;
            emits[l] = 0;
            if (i >= nsym) continue;
            uint32_t f = freq[sym[i]];
            if ((x[l] >> 20) >= f) {
                emits[l] = 1;
                k++;
            }
        }
        /* write the step's block, ascending lane order */
        uint32_t r = 0;
        for (uint32_t l = 0; l < lanes; l++) {
            if (!emits[l]) continue;
            rev[tail - k + r] = (uint16_t)(x[l] & 0xFFFFu);
            x[l] >>= 16;
            r++;
        }
        tail -= k;
        /* the state update */
        for (uint32_t l = 0; l < lanes; l++) {
            uint64_t i = (uint64_t)tt * lanes + l;
            if (i >= nsym) continue;
            uint32_t s = sym[i];
            uint32_t f = freq[s];
            x[l] = (x[l] / f) * OR_PROB_SCALE + (x[l] % f) + cum[s];
        }
    }
    uint32_t w = nsym - tail;
    for (uint32_t j = 0; j < w; j++) words_out[j] = rev[tail + j];
    for (uint32_t l = 0; l < lanes; l++) states_out[l] = x[l];
    *nwords_out = w;
    free(x); free(emits); free(rev);
    return OR_OK;
}

int oracle_rans_decode(const uint32_t *states_in, const uint16_t *words,
                       uint32_t nwords, uint32_t nsym, const uint16_t freq[256],
                       uint32_t lanes, uint8_t *sym_out) {
    if (lanes == 0 || lanes > 1024) return OR_ERR_INVALID_ARG;
    uint32_t cum[256];
    or_cumulative(freq, cum);
    if (cum[255] + freq[255] != OR_PROB_SCALE) return OR_ERR_CORRUPT;
    uint8_t owner[OR_PROB_SCALE];
    for (int s = 0; s < 256; s++)
        for (uint32_t j = cum[s]; j < cum[s] + freq[s]; j++) owner[j] = (uint8_t)s;

    uint32_t *x = (uint32_t *)malloc(sizeof(uint32_t) * lanes);
    if (!x) return OR_ERR_INVALID_ARG;
    for (uint32_t l = 0; l < lanes; l++) x[l] = states_in[l];
    uint32_t pos = 0;
    int status = OR_OK;
    uint32_t steps = (nsym + lanes - 1) / lanes;
    for (uint32_t t = 0; t < steps && status == OR_OK; t++) {
        for (uint32_t l = 0; l < lanes; l++) {
            uint64_t i = (uint64_t)t * lanes + l;
            if (i >= nsym) break;
            uint32_t slot = x[l] & (OR_PROB_SCALE - 1);
            uint32_t s = owner[slot];
            x[l] = freq[s] * (x[l] >> OR_PROB_BITS) + slot - cum[s];
            if (x[l] < OR_STATE_LOW) {
                if (pos >= nwords) {
                    status = OR_ERR_CORRUPT;
                    break;
                }
                x[l] = (x[l] << 16) | words[pos];
                pos++;
            }
            sym_out[i] = (uint8_t)s;
        }
    }
    if (status == OR_OK) {
        for (uint32_t l = 0; l < lanes; l++)
            if (x[l] != OR_STATE_LOW) status = OR_ERR_CORRUPT;
        if (pos != nwords) status = OR_ERR_CORRUPT;
    }
    free(x);
    return status;
}

/* ------------------------------------------------------------------ */
/* Accounting diagnostic.  For one chunk coded with 32 lanes:          */
/*  coded_bits = 16 w + sum over lanes of log2(x_final / 2^16)         */
/*  ideal_bits = sum over symbols of log2(4096 / f_s)                  */
/*  slack_bound = sum over symbols of -log2(1 - f_s / x_i)             */
/*              + sum over words of log2(1 + lo / (2^16 * hi))         */
/* where x_i is the state a symbol is coded from (after renormalising) */
/* and (hi, lo) are the two halves split by a renormalisation.  One     */
/* coding step maps x to x*4096/f times (1 + delta), |delta| < f/x, and */
/* one renormalisation divides x by 2^16 (1 + lo/(2^16 hi)), so         */
/* |coded_bits - ideal_bits| <= slack_bound exactly.                    */
/* ------------------------------------------------------------------ */
int oracle_chunk_accounting(const uint8_t *sym, uint32_t nsym,
                            const uint16_t freq[256], double *coded_bits,
                            double *ideal_bits, double *slack_bound) {
    uint32_t cum[256];
    or_cumulative(freq, cum);
    uint32_t x[OR_LANES];
    for (uint32_t l = 0; l < OR_LANES; l++) x[l] = OR_STATE_LOW;
    double ideal = 0.0, slack = 0.0;
    uint64_t w = 0;
    for (uint32_t ii = nsym; ii-- > 0;) {
        uint32_t l = ii % OR_LANES;
        uint32_t s = sym[ii];
        uint32_t f = freq[s];
        if (f == 0) return OR_ERR_INVALID_ARG;
        if ((x[l] >> 20) >= f) {
            uint32_t lo = x[l] & 0xFFFFu, hi = x[l] >> 16;
            slack += log2(1.0 + (double)lo / (65536.0 * (double)hi));
            x[l] = hi;
            w++;
        }
        ideal += log2((double)OR_PROB_SCALE / (double)f);
        slack += -log2(1.0 - (double)f / (double)x[l]);
        x[l] = (x[l] / f) * OR_PROB_SCALE + (x[l] % f) + cum[s];
    }
    double coded = 16.0 * (double)w;
    for (uint32_t l = 0; l < OR_LANES; l++) coded += log2((double)x[l] / 65536.0);
    *coded_bits = coded;
    *ideal_bits = ideal;
    *slack_bound = slack;
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Whole container: encode.                                            */
/* ------------------------------------------------------------------ */
int oracle_encode(const void *in, uint64_t n, int dtype, uint8_t *out,
                  uint64_t out_cap, uint64_t *out_size) {
    if (!or_dtype_ok(dtype)) return OR_ERR_INVALID_ARG;
    if (n > 0 && in == NULL) return OR_ERR_INVALID_ARG;
    if (out == NULL || out_size == NULL) return OR_ERR_INVALID_ARG;
    if (out_cap < oracle_encode_bound(n, dtype)) return OR_ERR_CAPACITY;

    or_layout lay;
    or_make_layout(n, dtype, &lay);
    memset(out, 0, lay.off_exp);

    /* 1. planes */
    uint8_t *expo = (uint8_t *)malloc(n > 0 ? n : 1);
    if (!expo) return OR_ERR_INVALID_ARG;
    if (dtype == OR_BF16)
        oracle_split_bf16((const uint16_t *)in, n, expo, out + lay.off_raw);
    else if (dtype == OR_FP16)
        oracle_split_fp16((const uint16_t *)in, n, expo, out + lay.off_raw);
    else if (dtype == OR_FP8E4M3)  /* the raw nibbles land in the zeroed section */
        oracle_split_fp8e4m3((const uint8_t *)in, n, expo, out + lay.off_raw);
    else if (dtype == OR_FP8E5M2)
        oracle_split_fp8e5m2((const uint8_t *)in, n, expo, out + lay.off_raw);
    else if (dtype == OR_BF16_HIGHBYTE)
        oracle_split_bf16_highbyte((const uint16_t *)in, n, expo, out + lay.off_raw);
    else
        oracle_split_fp32((const uint32_t *)in, n, expo, out + lay.off_sign,
                          out + lay.off_mant);

    /* 2. per-tensor histogram and 12-bit table */
    uint64_t counts[256];
    uint16_t freq[256];
    oracle_histogram(expo, n, counts);
    oracle_normalize(counts, freq);

    /* 3. chunks */
    uint32_t states[OR_LANES];
    uint16_t *words = (uint16_t *)malloc(sizeof(uint16_t) * OR_CHUNK_SYMBOLS);
    if (!words) { free(expo); return OR_ERR_INVALID_ARG; }
    uint64_t choff = 0;
    for (uint64_t k = 0; k < lay.nc; k++) {
        uint32_t nsym = or_chunk_nsym(n, k);
        const uint8_t *sym = expo + k * OR_CHUNK_SYMBOLS;
        uint32_t w = 0;
        oracle_rans_encode(sym, nsym, freq, OR_LANES, states, words, &w);
        uint64_t coded_len = 128u + 2u * (uint64_t)w;
        uint8_t *dst = out + lay.off_exp + choff;
        uint64_t len;
        if (coded_len < nsym) {
            len = coded_len;
            for (uint32_t l = 0; l < OR_LANES; l++) put_u32(dst + 4 * l, states[l]);
            for (uint32_t j = 0; j < w; j++) put_u16(dst + 128 + 2 * j, words[j]);
        } else {
            /* "do not shrink" -> raw; a tie goes raw */
            len = nsym;
            for (uint32_t j = 0; j < nsym; j++) dst[j] = sym[j];
        }
        for (uint64_t j = len; j < round_up16(len); j++) dst[j] = 0;
        put_u64(out + lay.off_chunk_off + 8 * k, choff);
        put_u32(out + lay.off_chunk_len + 4 * k, (uint32_t)len);
        choff += round_up16(len);
    }
    put_u64(out + lay.off_chunk_off + 8 * lay.nc, choff);
    free(words);
    free(expo);

    /* 4. header and table */
    out[0] = 'W'; out[1] = 'C'; out[2] = 'Z'; out[3] = '1';
    put_u16(out + 4, 1);
    out[6] = (uint8_t)dtype;
    out[7] = (uint8_t)OR_LANES;
    put_u64(out + 8, n);
    put_u32(out + 16, OR_CHUNK_SYMBOLS);
    put_u32(out + 20, (uint32_t)lay.nc);
    put_u16(out + 24, OR_PROB_BITS);
    put_u16(out + 26, 0);
    put_u32(out + 28, 0);
    put_u64(out + 32, lay.off_raw);
    put_u64(out + 40, lay.off_exp);
    put_u64(out + 48, choff);
    put_u64(out + 56, lay.off_exp + choff);
    for (int s = 0; s < 256; s++) put_u16(out + OR_FREQ_OFFSET + 2 * s, freq[s]);
    *out_size = lay.off_exp + choff;
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Whole container: validation and decode.                             */
/* ------------------------------------------------------------------ */
typedef struct {
    or_layout lay;
    int dtype;
    uint16_t freq[256];
} or_header;

/* Checks everything that does not need the coded words. */
static int or_parse(const uint8_t *c, uint64_t bytes, or_header *h) {
    if (c == NULL || bytes < OR_CHUNK_OFF_OFFSET + 8) return OR_ERR_CORRUPT;
    if (c[0] != 'W' || c[1] != 'C' || c[2] != 'Z' || c[3] != '1') return OR_ERR_CORRUPT;
    if (get_u16(c + 4) != 1) return OR_ERR_CORRUPT;
    int dtype = c[6];
    if (!or_dtype_ok(dtype)) return OR_ERR_CORRUPT;
    if (c[7] != OR_LANES) return OR_ERR_CORRUPT;
    uint64_t n = get_u64(c + 8);
    if (get_u32(c + 16) != OR_CHUNK_SYMBOLS) return OR_ERR_CORRUPT;
    if (get_u16(c + 24) != OR_PROB_BITS) return OR_ERR_CORRUPT;
    if (get_u16(c + 26) != 0 || get_u32(c + 28) != 0) return OR_ERR_CORRUPT;
    if (n > (1ull << 47)) return OR_ERR_CORRUPT;
    or_make_layout(n, dtype, &h->lay);
    h->dtype = dtype;
    if (get_u32(c + 20) != h->lay.nc) return OR_ERR_CORRUPT;
    if (get_u64(c + 32) != h->lay.off_raw) return OR_ERR_CORRUPT;
    if (get_u64(c + 40) != h->lay.off_exp) return OR_ERR_CORRUPT;
    if (bytes < h->lay.off_exp) return OR_ERR_CORRUPT;
    uint64_t exp_bytes = get_u64(c + 48);
    uint64_t total = get_u64(c + 56);
    if (total != h->lay.off_exp + exp_bytes || total > bytes) return OR_ERR_CORRUPT;

    uint32_t sum = 0;
    for (int s = 0; s < 256; s++) {
        h->freq[s] = get_u16(c + OR_FREQ_OFFSET + 2 * s);
        sum += h->freq[s];
    }
    if (n == 0 ? sum != 0 : sum != OR_PROB_SCALE) return OR_ERR_CORRUPT;

    if (get_u64(c + h->lay.off_chunk_off) != 0) return OR_ERR_CORRUPT;
    for (uint64_t k = 0; k < h->lay.nc; k++) {
        uint32_t nsym = or_chunk_nsym(n, k);
        uint32_t len = get_u32(c + h->lay.off_chunk_len + 4 * k);
        uint64_t o0 = get_u64(c + h->lay.off_chunk_off + 8 * k);
        uint64_t o1 = get_u64(c + h->lay.off_chunk_off + 8 * (k + 1));
        int raw = (len == nsym);
        int coded = (len >= 128 && len < nsym && (len - 128) % 2 == 0);
        if (!raw && !coded) return OR_ERR_CORRUPT;
        if (o1 != o0 + round_up16(len)) return OR_ERR_CORRUPT;
    }
    if (get_u64(c + h->lay.off_chunk_off + 8 * h->lay.nc) != exp_bytes) return OR_ERR_CORRUPT;
    return OR_OK;
}

int oracle_read_header(const uint8_t *cont, uint64_t cont_bytes, uint64_t *n,
                       int *dtype, uint64_t *nchunks) {
    or_header h;
    int st = or_parse(cont, cont_bytes, &h);
    if (st != OR_OK) return st;
    *n = h.lay.n;
    *dtype = h.dtype;
    *nchunks = h.lay.nc;
    return OR_OK;
}

/* Decodes chunk k of a parsed container into values [0, nsym) of out_vals
 * (which points at the output slot of the chunk's first value). */
static int or_decode_one_chunk(const uint8_t *c, const or_header *h, uint64_t k,
                               uint8_t *expo, uint16_t *words, void *out_vals) {
    uint64_t n = h->lay.n;
    uint32_t nsym = or_chunk_nsym(n, k);
    uint32_t len = get_u32(c + h->lay.off_chunk_len + 4 * k);
    uint64_t o0 = get_u64(c + h->lay.off_chunk_off + 8 * k);
    const uint8_t *src = c + h->lay.off_exp + o0;

    if (len == nsym) {
        for (uint32_t j = 0; j < nsym; j++) expo[j] = src[j];
    } else {
        uint32_t states[OR_LANES];
        uint32_t w = (len - 128) / 2;
        for (uint32_t l = 0; l < OR_LANES; l++) states[l] = get_u32(src + 4 * l);
        for (uint32_t j = 0; j < w; j++) words[j] = get_u16(src + 128 + 2 * j);
        int st = oracle_rans_decode(states, words, w, nsym, h->freq, OR_LANES, expo);
        if (st != OR_OK) return st;
    }

    /* re-merge the planes into the original bits */
    uint64_t first = k * OR_CHUNK_SYMBOLS;
    for (uint32_t j = 0; j < nsym; j++) {
        uint64_t i = first + j;
        if (h->dtype == OR_BF16) {
            uint8_t sm = c[h->lay.off_raw + i];
            uint16_t sign = (uint16_t)((sm >> 7) & 1u);
            uint16_t mant = (uint16_t)(sm & 0x7Fu);
            ((uint16_t *)out_vals)[j] = (uint16_t)((sign << 15) | ((uint16_t)expo[j] << 7) | mant);
        } else if (h->dtype == OR_FP16) {
            /* undo the byte split, then the reorder E S M -> S E M */
            uint16_t r = (uint16_t)(((uint16_t)expo[j] << 8) | c[h->lay.off_raw + i]);
            uint16_t e5 = (uint16_t)(r >> 11);
            uint16_t sign = (uint16_t)((r >> 10) & 1u);
            uint16_t mant = (uint16_t)(r & 0x3FFu);
            ((uint16_t *)out_vals)[j] = (uint16_t)((sign << 15) | (e5 << 10) | mant);
        } else if (h->dtype == OR_FP8E4M3) {
            /* undo the nibble split, then the reorder E S M -> S E M */
            uint8_t lo = (uint8_t)((c[h->lay.off_raw + i / 2] >> (i % 2 ? 4 : 0)) & 0xFu);
            uint8_t r = (uint8_t)((expo[j] << 4) | lo);
            uint8_t e4 = (uint8_t)(r >> 4);
            uint8_t sign = (uint8_t)((r >> 3) & 1u);
            uint8_t mant = (uint8_t)(r & 7u);
            ((uint8_t *)out_vals)[j] = (uint8_t)((sign << 7) | (e4 << 3) | mant);
        } else if (h->dtype == OR_FP8E5M2) {
            uint8_t lo = (uint8_t)((c[h->lay.off_raw + i / 2] >> (i % 2 ? 4 : 0)) & 0xFu);
            uint8_t r = (uint8_t)((expo[j] << 4) | lo);
            uint8_t e5 = (uint8_t)(r >> 3);
            uint8_t sign = (uint8_t)((r >> 2) & 1u);
            uint8_t mant = (uint8_t)(r & 3u);
            ((uint8_t *)out_vals)[j] = (uint8_t)((sign << 7) | (e5 << 2) | mant);
        } else if (h->dtype == OR_BF16_HIGHBYTE) {
            ((uint16_t *)out_vals)[j] = (uint16_t)(((uint16_t)expo[j] << 8) | c[h->lay.off_raw + i]);
        } else {
            uint32_t sign = (c[h->lay.off_sign + i / 8] >> (i % 8)) & 1u;
            const uint8_t *m = c + h->lay.off_mant + 3 * i;
            uint32_t mant = ((uint32_t)m[0] | ((uint32_t)m[1] << 8) | ((uint32_t)m[2] << 16)) & 0x7FFFFFu;
            ((uint32_t *)out_vals)[j] = (sign << 31) | ((uint32_t)expo[j] << 23) | mant;
        }
    }
    return OR_OK;
}

int oracle_decode(const uint8_t *cont, uint64_t cont_bytes, void *out,
                  uint64_t out_cap) {
    or_header h;
    int st = or_parse(cont, cont_bytes, &h);
    if (st != OR_OK) return st;
    uint64_t elem = or_elem(h.dtype);
    if (h.lay.n * elem > out_cap) return OR_ERR_CAPACITY;
    if (h.lay.n > 0 && out == NULL) return OR_ERR_INVALID_ARG;
    uint8_t *expo = (uint8_t *)malloc(OR_CHUNK_SYMBOLS);
    uint16_t *words = (uint16_t *)malloc(sizeof(uint16_t) * OR_CHUNK_SYMBOLS);
    if (!expo || !words) { free(expo); free(words); return OR_ERR_INVALID_ARG; }
    for (uint64_t k = 0; k < h.lay.nc && st == OR_OK; k++) {
        uint8_t *dst = (uint8_t *)out + k * OR_CHUNK_SYMBOLS * elem;
        st = or_decode_one_chunk(cont, &h, k, expo, words, dst);
    }
    free(expo);
    free(words);
    return st;
}

int oracle_decode_chunk(const uint8_t *cont, uint64_t cont_bytes, uint64_t k,
                        void *out, uint64_t out_cap) {
    or_header h;
    int st = or_parse(cont, cont_bytes, &h);
    if (st != OR_OK) return st;
    if (k >= h.lay.nc) return OR_ERR_INVALID_ARG;
    uint64_t elem = or_elem(h.dtype);
    if ((uint64_t)or_chunk_nsym(h.lay.n, k) * elem > out_cap) return OR_ERR_CAPACITY;
    if (out == NULL) return OR_ERR_INVALID_ARG;
    uint8_t *expo = (uint8_t *)malloc(OR_CHUNK_SYMBOLS);
    uint16_t *words = (uint16_t *)malloc(sizeof(uint16_t) * OR_CHUNK_SYMBOLS);
    if (!expo || !words) { free(expo); free(words); return OR_ERR_INVALID_ARG; }
    st = or_decode_one_chunk(cont, &h, k, expo, words, out);
    free(expo);
    free(words);
    return st;
}

/* ---------------------------------------------------------------------------
 * CRC-32, one bit at a time: the register holds the remainder with the
 * coefficient of x^31 in bit 0 (bits are taken least significant first), so
 * a step shifts right and, when a 1 falls out, subtracts (xors) the generator
 * without its x^32 term, written in that same reversed order: 0xEDB88320. */
uint32_t oracle_crc32(const uint8_t *data, uint64_t bytes) {
    const uint32_t gen_reversed = 0xEDB88320u;
    uint32_t r = 0xFFFFFFFFu;
    for (uint64_t i = 0; i < bytes; i++) {
        r ^= data[i];
        for (int b = 0; b < 8; b++)
            r = (r & 1u) ? (r >> 1) ^ gen_reversed : (r >> 1);
    }
    return r ^ 0xFFFFFFFFu;
}

int oracle_crc32_blocks(const uint8_t *data, uint64_t bytes, uint64_t block_bytes,
                        uint32_t *crc) {
    if (block_bytes == 0 || (bytes > 0 && (data == NULL || crc == NULL)))
        return OR_ERR_INVALID_ARG;
    for (uint64_t i = 0; i * block_bytes < bytes; i++) {
        uint64_t len = bytes - i * block_bytes;
        if (len > block_bytes) len = block_bytes;
        crc[i] = oracle_crc32(data + i * block_bytes, len);
    }
    return OR_OK;
}
