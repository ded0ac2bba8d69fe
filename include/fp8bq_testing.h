/*
 * fp8bq_testing.h -- test hooks of libfp8bq.so.  Not part of the product
 * interface: no product path calls them, and a user of the library has no
 * reason to.  They exist so that the library's failure handling can be
 * exercised on a GPU without faulting it.
 */
#ifndef FP8BQ_TESTING_H
#define FP8BQ_TESTING_H

#include <stdint.h>

#include "fp8bq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fp8bq_gemm_ws with one of its CTA pairs made to withhold its split-tile
 * flags, and every bounded wait of the launch limited to wait_limit_ns.
 * There is no counterpart on the pages: it tests the split-tile schedule's
 * bounded wait (the one wait that depends on other CTA pairs), not the
 * method.
 *   withhold_pair  CTA pair (cluster index) whose split-tile piece stores its
 *                  FP32 partial sum into its workspace slot as usual but never
 *                  raises the slot's flags.  When that pair holds a piece that
 *                  does not start at the tile's first K block, the tile's head
 *                  piece waits for those flags until the limit expires: the
 *                  kernel then records FP8BQ_ERR_TIMEOUT in the device status
 *                  word, stops early (the launch's output is undefined) and
 *                  releases its tensor memory; fp8bq_check() reports it.
 *                  When that pair holds no such piece, the call is
 *                  fp8bq_gemm_ws.
 *   wait_limit_ns  the limit of every bounded wait in this launch, in
 *                  [100000, 2000000000] ns (the product limit is 2 s).
 *   workspace      required (non-NULL), as for fp8bq_gemm_ws.  After a call
 *                  that timed out, zero the workspace before its next use,
 *                  as fp8bq_gemm_ws's contract asks after any failure.
 * Errors: those of fp8bq_gemm_ws; ERR_INVALID_ARG for a NULL workspace, a
 * negative withhold_pair or a limit outside the range above.
 */
int fp8bq_testing_gemm_ws_withhold(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
                                   int64_t K, int64_t ldd, uint32_t flags, void* workspace, int64_t workspace_bytes,
                                   int withhold_pair, int64_t wait_limit_ns, fp8bq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8BQ_TESTING_H */
