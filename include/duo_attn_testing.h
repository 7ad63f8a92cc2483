/*
 * duo_attn_testing.h -- failure-injection hook of libduoattn.so, for tests of
 * the failure-detection path only.
 *
 * Every wait inside the library's pipelined kernels (a consumer waiting for a
 * tile, a producer waiting for a free stage) is bounded: when one expires the
 * kernel records DUO_ERR_TIMEOUT in the device status word, stops, and
 * returns, so the CUDA context stays usable.  This hook makes such a wait
 * expire on purpose without faulting or hanging the GPU: the tile producer of
 * CTA 0 of the selected kernel issues no copy from its `tile`-th tile on, so
 * the consumers' waits for it run out (about two seconds) and the call's
 * status reads DUO_ERR_TIMEOUT.  No copy is left in flight.
 *
 * The setting is process-wide and stays until it is changed; the default (and
 * tile = -1) is off.  Nothing in a production path sets it.  Not part of the
 * method on the pages: this is a test interface.
 */
#ifndef DUO_ATTN_TESTING_H
#define DUO_ATTN_TESTING_H

#include <stdint.h>

#include "duo_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

#define DUO_TESTING_DECODE 1        /* decode_split (duo_attn_decode, _static)   */
#define DUO_TESTING_PREFILL 2       /* prefill_fwd (duo_attn_prefill)            */
#define DUO_TESTING_DECODE_BLOCK 3  /* decode_block_split (duo_attn_decode_block) */

/* Withholds tile `tile` (counted over CTA 0's producer loop, from 0) and every
 * later one in the selected kernel's launches from now on; tile = -1 turns it
 * off.  Returns DUO_OK, or DUO_ERR_INVALID_ARG for an unknown kernel or a
 * tile below -1. */
DUO_API int duo_testing_withhold_tile(int32_t kernel, int32_t tile);

/* The prefill's exponential on the FMA pipe (2^x by Cody-Waite range
 * reduction and a degree-3 polynomial, see ex2_poly2 in the sources), applied
 * to n fp32 values: y[i] = 2^x[i].  x, y: device fp32 [n], 16-byte aligned.
 * Inputs below -125 give about 2^-125.  For tests of its error bound against
 * the exact 2^x; asynchronous on `stream`.  DUO_ERR_INVALID_ARG for NULL or
 * misaligned pointers or n < 0. */
DUO_API int duo_testing_ex2(const float *x, float *y, int64_t n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DUO_ATTN_TESTING_H */
