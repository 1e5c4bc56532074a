/*
 * wc_diag.h -- self-checks of the B200 weight codec's arithmetic, for tests.
 *
 * The rANS coding step of the encoder ("SMEF -- blog companion code",
 * pass4_rans.py; "PTWM", How it works 2) divides the state x by the
 * symbol's frequency f.  The library computes x / f with multiplies (a
 * 32-bit multiplier and a shift when every frequency of a tensor is at most
 * 2048, a 64-bit multiplier otherwise) and relies on a proof that the result
 * is exact for every state it divides: 16 f <= x < f 2^20 (states are
 * >= 2^16 before a step, and one at or above f 2^20 first loses 16 bits).  This call checks that
 * claim exhaustively on the device, with the same device function the
 * encoder runs.
 */
#ifndef WC_DIAG_H
#define WC_DIAG_H

#include <stdint.h>

#include "wc.h"

#ifdef __cplusplus
extern "C" {
#endif

/* For every f in [f_first, f_last] and every state x in [16 f, f 2^20), compare
 * the coding step (the table entry of f with cumulative frequency 0, in the
 * narrow format if wide == 0, else the wide one) with x / f * 4096 + x % f.
 *   wide      0: the 32-bit multiplier format, f_last <= 2048;
 *             1: the 64-bit format, f_last <= 4095.
 *   d_result  device, two uint64 (8-byte aligned), cleared by the call:
 *             [0] the number of mismatching (f, x), [1] one of them as
 *             f << 32 | x (0 if none).
 * Queued on `stream` (about 2^20 f states per f: the full ranges take a few
 * seconds).  Returns WC_OK, WC_ERR_INVALID_ARG or WC_ERR_CUDA. */
WC_API int32_t wc_check_coder_division(int32_t wide, uint32_t f_first, uint32_t f_last,
                                       uint64_t *d_result, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* WC_DIAG_H */
