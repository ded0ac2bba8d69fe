/*
 * fp8bq.h -- C ABI of the blockwise-FP8 linear layer for NVIDIA B200 (sm_100a).
 *
 * The method (page titles and sections):
 *   "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090" (agihunt
 *   paper digest), section "方法": Transformer linear layers are trained in
 *   blockwise FP8 from random init, activations grouped by 128, weights in
 *   128x128 blocks, MXFP8 on Blackwell, master weights and optimizer state kept
 *   in BF16/FP32; section "术语", entry "blockwise FP8": one scale per local
 *   block so that an outlier cannot blow up a single per-tensor scale.
 *   "清华开源 Puro-2B" (ModelScope community post), section
 *   "精度：FP8 分块量化与净效率收益": the main linear layers' matmuls run in FP8
 *   (fine-grained block quantization in the manner of DeepSeek-V3).
 *
 * Conventions shared by every call:
 *   - All data pointers are DEVICE pointers to caller-owned memory.  The library
 *     allocates no device memory and never frees caller memory (the one array
 *     it owns, fp8bq_gemm_noalloc's workspace, is part of the loaded library).
 *   - Every compute call is asynchronous on `stream` (NULL = legacy default
 *     stream) and never synchronizes; errors it can see at launch are returned
 *     at once, errors that happen on the device surface at fp8bq_check().
 *   - Matrices are row-major; every `ld*` is a leading dimension in ELEMENTS.
 *   - FP8 data is OCP E4M3FN (bias 7, max 448, no infinities).  BF16 inputs
 *     must be finite.
 *   - Scale arrays (a library choice; the pages fix none):
 *       1x128 row groups of an operand with R rows and contraction length C:
 *         scales[cb * fp8bq_row_scale_ld(R) + r], cb = k / 128; the row
 *         stride is R rounded up to a multiple of 128 and the pad entries
 *         r >= R hold the neutral scale (1.0f, or the byte 127);
 *       128x128 blocks of W [N,K]: scales[kb * ceil(N/128) + nb];
 *       1x32 row groups (MX blocks, the other reading of "MXFP8 on
 *         Blackwell": the OCP Microscaling format's 32-value blocks with
 *         E8M0 scales): as 1x128 row groups with cb = k / 32.
 *     FP32 scales are `float`; UE8M0 scales are one byte e + 127 meaning 2^e.
 *   - Scale definitions:  FP32: s = fl32(amax / 448) (s = 1 for an all-zero
 *     group), code q = E4M3_RNE_satfinite(fl32(x / s)).  UE8M0: e = the least
 *     integer with amax <= 448 * 2^e, clamped to [-127, 127] (e = 0 for an
 *     all-zero group), q = E4M3_RNE_satfinite(x * 2^-e).
 *   - Return value: FP8BQ_OK or one of the negative FP8BQ_ERR_* codes.  A call
 *     that returns an error has launched no kernel and written no caller
 *     memory.  (The one exception: when fp8bq_gemm_noalloc's launch itself
 *     fails with ERR_CUDA, the clearing of its own array's flags has
 *     already been queued; argument errors queue nothing.)
 */
#ifndef FP8BQ_H
#define FP8BQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* fp8bq_stream_t;

#define FP8BQ_OK 0
#define FP8BQ_ERR_INVALID_ARG (-1) /* null pointer or unknown enum value            */
#define FP8BQ_ERR_SHAPE (-2)       /* bad dimension (see each call)                 */
#define FP8BQ_ERR_ALIGN (-3)       /* pointer or leading dimension not 16-B aligned */
#define FP8BQ_ERR_UNSUPPORTED (-4) /* no sm_100 device, or an operand combination   */
                                   /* this library does not build                   */
#define FP8BQ_ERR_CUDA (-5)        /* a CUDA call failed; see fp8bq_last_cuda_error */
#define FP8BQ_ERR_TIMEOUT (-6)     /* a bounded wait inside a kernel expired        */

typedef enum { FP8BQ_SCALE_FP32 = 0, FP8BQ_SCALE_UE8M0 = 1 } fp8bq_scale_fmt;
typedef enum {
  FP8BQ_GRAN_ROW_1x128 = 0,
  FP8BQ_GRAN_BLOCK_128x128 = 1,
  FP8BQ_GRAN_ROW_1x32 = 2 /* MX blocks: 32 consecutive contraction values, UE8M0 only */
} fp8bq_gran;
typedef enum { FP8BQ_E4M3 = 0, FP8BQ_BF16 = 1 } fp8bq_dtype;

/* fp8bq_gemm flags */
#define FP8BQ_GEMM_ACCUMULATE_F32 1u /* D is FP32 and D += A B^T */

/* fp8bq_swiglu_quantize: OR into fmt to round h once from its exact value */
#define FP8BQ_SWIGLU_EXACT 0x100

/*
 * One GEMM operand, seen as a logical matrix [rows, C] whose second index runs
 * over the contraction C.
 *   data     E4M3 codes (dtype E4M3), or BF16 values (dtype BF16: operand A
 *            only, quantized inside the GEMM with 1x128 groups and format
 *            `fmt`, bit-identical to fp8bq_quantize_act).
 *   ld       leading dimension in elements; ld * element size % 16 == 0.
 *   k_major  1: element (r, k) is data[r*ld + k] (contraction contiguous);
 *            0: element (r, k) is data[k*ld + r] (rows contiguous).  k_major = 0
 *            is accepted for a 128x128-block operand B (the dgrad GEMM reads
 *            W [N,K] as W^T this way, without a transpose pass).
 *   scales   scale array (ignored when dtype is BF16).
 *   gran     FP8BQ_GRAN_ROW_1x128 (A, or B in the weight-gradient GEMM),
 *            FP8BQ_GRAN_BLOCK_128x128 (B only), or FP8BQ_GRAN_ROW_1x32 (MX:
 *            A and B both, k_major, UE8M0; the weight is quantized in 1x32
 *            groups along its contraction like an activation).
 *   fmt      FP8BQ_SCALE_FP32 or FP8BQ_SCALE_UE8M0, per operand.  Both
 *            UE8M0: the block-scaled MMA.  Otherwise (both FP32, or a mixed
 *            pair) the per-128-K promotion path, in which a UE8M0 operand's
 *            scale bytes are decoded to the FP32 value 2^e as they are
 *            staged; the product is the same definition either way.  A BF16
 *            A is quantized in its own fmt and B must then have the same.
 *   s_stride_k, s_stride_r
 *            the scale of element (r, k) is scales[(k/G)*s_stride_k +
 *            t*s_stride_r], t = r (row groups) or t = r/128 (blocks), G = 32
 *            for FP8BQ_GRAN_ROW_1x32 and 128 otherwise.  Row
 *            groups need s_stride_r == 1 and s_stride_k a multiple of 128;
 *            blocks are either (ceil(rows/128), 1) or, for W^T, (1, C/128).
 */
typedef struct fp8bq_operand {
  const void* data;
  int64_t ld;
  int32_t dtype;
  int32_t k_major;
  const void* scales;
  int32_t gran;
  int32_t fmt;
  int64_t s_stride_k;
  int64_t s_stride_r;
} fp8bq_operand;

/*
 * 1x128 activation quantization ("方法": activations grouped by 128).
 *   x       BF16 [M, K], leading dimension ldx (ldx >= K, ldx % 8 == 0).
 *   q       E4M3 [M, K], leading dimension K.
 *   scales  [K/128][fp8bq_row_scale_ld(M)] of float (FP32) or uint8 (UE8M0).
 * Each row's K values form K/128 groups of 128 consecutive columns.
 * Errors: ERR_INVALID_ARG (null pointer, bad fmt), ERR_SHAPE (M < 0, K < 0,
 * K % 128 != 0, ldx < K), ERR_ALIGN (x, q or scales not 16-B aligned, or
 * ldx % 8 != 0).  M == 0 or K == 0 is a no-op.
 */
int fp8bq_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                       int fmt, fp8bq_stream_t stream);

/*
 * 1x128 quantization along the token dimension, for the weight-gradient GEMM
 * that contracts over tokens: the act quantizer applied to X^T.
 *   x       BF16 [M, K], leading dimension ldx.
 *   qt      E4M3 [K, M], leading dimension M (the transpose of the codes).
 *   scales  [M/128][fp8bq_row_scale_ld(K)].
 * Errors: as fp8bq_quantize_act, with ERR_SHAPE when M % 128 != 0 (M is the
 * contraction here) and ERR_ALIGN when K % 8 != 0 or ldx % 8 != 0.
 */
int fp8bq_quantize_act_t(const void* x, int64_t M, int64_t K, int64_t ldx, void* qt, void* scales,
                         int fmt, fp8bq_stream_t stream);

/*
 * Both activation layouts from one read of X: exactly the outputs of
 * fp8bq_quantize_act (q, scales) and fp8bq_quantize_act_t (qt, scales_t) on
 * the same x, bit for bit.  Training needs both for each linear layer's input
 * (forward and weight gradient) and for its output gradient (data gradient
 * and weight gradient); this call reads the BF16 tensor once instead of twice.
 * The pages have no such call; it is the same method, fused.
 *   x         BF16 [M, K], leading dimension ldx.
 *   q         E4M3 [M, K] (ld K); scales [K/128][fp8bq_row_scale_ld(M)].
 *   qt        E4M3 [K, M] (ld M); scales_t [M/128][fp8bq_row_scale_ld(K)].
 * Errors: ERR_SHAPE when K % 128 != 0 or M % 128 != 0; otherwise as
 * fp8bq_quantize_act.
 */
int fp8bq_quantize_act_dual(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                            void* qt, void* scales_t, int fmt, fp8bq_stream_t stream);

/*
 * SwiGLU fused with the quantization of its output: the down projection's
 * input produced and quantized in one pass, without a BF16 round trip
 * through HBM.  The pages keep the activation function outside the FP8
 * matmuls ("清华开源 Puro-2B", section "精度"; the digest's "方法": a
 * Qwen3-1.7B-like model, whose MLP is SwiGLU); this call has no counterpart
 * on the pages beyond computing that BF16 activation and quantizing it.
 *   gu        BF16 [M, 2F], leading dimension ldgu: [gate | up], the gate/up
 *             GEMM's output with the two halves side by side.
 *   h         optional BF16 [M, F] (ld F): h = silu(gate) * up =
 *             gate * up / (1 + e^-gate) in FP32, rounded to BF16 (nearest,
 *             ties to even); may be NULL.  Within one BF16 ulp of the exact
 *             value (while gate * up stays below the FP32 maximum); with
 *             FP8BQ_SWIGLU_EXACT in fmt, the exact value rounded
 *             once to BF16 (nearest, ties to even): the FP32 value where its
 *             error bound decides the rounding, float64 (the definition's
 *             order, (gate / (1 + e^-gate)) * up) for the rest; ~60% more
 *             time.
 *   q, scales h quantized as fp8bq_quantize_act (1x128 groups along F) of
 *             exactly that BF16 h: E4M3 [M, F] (ld F), scales
 *             [F/128][fp8bq_row_scale_ld(M)].
 *   qt, scales_t  optional (both or neither): h quantized as
 *             fp8bq_quantize_act_t: [F, M] (ld M), [M/128][fp8bq_row_scale_ld(F)].
 *   fmt       FP8BQ_SCALE_FP32 or FP8BQ_SCALE_UE8M0, optionally OR
 *             FP8BQ_SWIGLU_EXACT.
 * Errors: ERR_INVALID_ARG (null gu, q or scales; only one of qt, scales_t;
 * bad fmt), ERR_SHAPE (F % 128 != 0; M % 128 != 0 with qt; ldgu < 2F),
 * ERR_ALIGN (as fp8bq_quantize_act, and h, qt, scales_t 16-B aligned).
 */
int fp8bq_swiglu_quantize(const void* gu, int64_t M, int64_t F, int64_t ldgu, void* h, void* q, void* scales,
                          void* qt, void* scales_t, int fmt, fp8bq_stream_t stream);

/*
 * RMSNorm fused with the quantization of its output: the QKV and gate/up
 * projections' input produced and quantized without a BF16 round trip
 * through HBM.  The pages keep normalization outside the FP8 matmuls, in
 * BF16/FP32 ("清华开源 Puro-2B", section "精度"; the digest's "方法": a
 * Qwen3-1.7B-like model, whose blocks normalize with RMSNorm before these
 * projections); this call computes that BF16 output and quantizes it.
 *   x         BF16 [M, K], leading dimension ldx.
 *   gamma     BF16 [K], the norm's weight (16-byte aligned).
 *   eps       added to the mean square (finite, >= 0; Qwen3 uses 1e-6).
 *   rstd      FP32 [M], written: 1 / sqrt(mean_k x[r,k]^2 + eps), IEEE square
 *             root and division of the FP32 mean square (the value the norm's
 *             backward pass needs).
 *   h         optional BF16 [M, K] (ld K): h = x * rstd * gamma in FP32,
 *             rounded to BF16 (nearest, ties to even); may be NULL.  Within
 *             one BF16 ulp of the exact value.
 *   q, scales h quantized as fp8bq_quantize_act of exactly that BF16 h:
 *             E4M3 [M, K] (ld K), scales [K/128][fp8bq_row_scale_ld(M)].
 *   qt, scales_t  optional (both or neither): h quantized as
 *             fp8bq_quantize_act_t: [K, M] (ld M), [M/128][fp8bq_row_scale_ld(K)].
 *   fmt       FP8BQ_SCALE_FP32 or FP8BQ_SCALE_UE8M0.
 * Two launches on the stream: the row statistics, then the quantizer.
 * Errors: ERR_INVALID_ARG (null x, gamma, rstd, q or scales; only one of qt,
 * scales_t; bad fmt or eps), ERR_SHAPE (K % 128 != 0; M % 128 != 0 with qt),
 * ERR_ALIGN (as fp8bq_quantize_act; gamma, h, qt, scales_t 16-B aligned;
 * rstd 4-B aligned).
 */
int fp8bq_rmsnorm_quantize(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
                           float* rstd, void* h, void* q, void* scales, void* qt, void* scales_t, int fmt,
                           fp8bq_stream_t stream);

/*
 * fp8bq_rmsnorm_quantize with h rounded once from its exact value, so that
 * h, codes and scales equal the float64 definition's bit for bit.
 *   eps       added to the mean square (finite, >= 0), in double.
 *   rstd      float64 [M] (8-byte aligned), written: 1 / sqrt(mean_k x[r,k]^2
 *             + eps) in IEEE double (each square exact, the sum in double).
 *   h         optional BF16 [M, K] (ld K): x * rstd * gamma rounded once to
 *             BF16 (nearest, ties to even) from the exact product: the FP32
 *             products (of x, rstd rounded to FP32, and gamma) where their
 *             error bound (3 ulp) keeps every BF16 rounding boundary out of
 *             reach, float64 ((x * rstd) * gamma) for the rest.
 *   the other arguments and the errors as fp8bq_rmsnorm_quantize
 *   (ERR_ALIGN for an rstd not 8-byte aligned).
 */
int fp8bq_rmsnorm_quantize_exact(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, double eps,
                                 double* rstd, void* h, void* q, void* scales, void* qt, void* scales_t, int fmt,
                                 fp8bq_stream_t stream);

/*
 * MX-block quantization (1x32 groups, UE8M0 scales): the other reading of
 * "MXFP8 on Blackwell" ("方法"), with the OCP Microscaling format's 32-value
 * blocks in place of the 1x128 groups.  Same definitions as the calls above
 * with 32 for 128; the scale format is always UE8M0.
 *   fp8bq_quantize_act_mx:    x [M, K] -> q [M, K] (ld K), scales
 *                             [K/32][fp8bq_row_scale_ld(M)] (bytes); K % 128 == 0.
 *   fp8bq_quantize_act_t_mx:  x [M, K] -> qt [K, M] (ld M), scales
 *                             [M/32][fp8bq_row_scale_ld(K)]; M % 128 == 0, K % 8 == 0.
 *   fp8bq_quantize_act_dual_mx: both, from one read; K % 128 == 0, M % 128 == 0.
 * A weight W [N, K] takes fp8bq_quantize_act_mx for the forward GEMM and
 * fp8bq_quantize_act_t_mx (groups along N) for the data-gradient GEMM, since
 * 1x32 blocks, unlike 128x128 ones, depend on the orientation.
 * Errors: as fp8bq_quantize_act / _act_t / _act_dual.
 */
int fp8bq_quantize_act_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                          fp8bq_stream_t stream);
int fp8bq_quantize_act_t_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* qt, void* scales,
                            fp8bq_stream_t stream);
int fp8bq_quantize_act_dual_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                               void* qt, void* scales_t, fp8bq_stream_t stream);

/*
 * 128x128 weight-block quantization ("方法": weights in 128x128 blocks).
 *   w       BF16 [N, K], leading dimension ldw (ldw >= K, ldw % 8 == 0).
 *   q       E4M3 [N, K], leading dimension K.
 *   scales  [K/128][ceil(N/128)].  A block at the edge (N % 128 != 0) covers
 *           only its valid rows.
 * Errors: ERR_SHAPE when K % 128 != 0; otherwise as fp8bq_quantize_act.
 */
int fp8bq_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw, void* q, void* scales,
                          int fmt, fp8bq_stream_t stream);

/*
 * Several quantizations in one launch.  The pages have no such call: it is
 * the calls above (fp8bq_quantize_act / _act_t / _act_dual /
 * fp8bq_quantize_weight), run together by one persistent kernel over the
 * concatenated tiles of all jobs, so that the small tensors of a layer (its
 * weight and its input, say) share one pipeline ramp and one tail instead of
 * paying for one each.  Every job's outputs are bit-identical to those of
 * the single call of its kind on the same arguments.
 *   kind      FP8BQ_QUANT_ACT (q, scales), FP8BQ_QUANT_ACT_T (qt, scales_t),
 *             FP8BQ_QUANT_ACT_DUAL (all four), FP8BQ_QUANT_WEIGHT (q, scales
 *             as fp8bq_quantize_weight: 128x128 blocks of a weight [rows, cols],
 *             scales [cols/128][ceil(rows/128)]).  Pointers a kind does not use
 *             are ignored.
 *   x, rows, cols, ldx   the BF16 input and its shape, as in the single call.
 *   njobs     1 to 8; fmt, the scale format of every job.  A job with rows
 *             or cols 0 is skipped.
 * Errors: those of the single calls, per job (the first failing job's);
 * ERR_INVALID_ARG for a NULL jobs array, njobs outside 1..8 or an unknown kind.
 */
typedef enum {
  FP8BQ_QUANT_ACT = 0,
  FP8BQ_QUANT_ACT_T = 1,
  FP8BQ_QUANT_ACT_DUAL = 2,
  FP8BQ_QUANT_WEIGHT = 3
} fp8bq_quant_kind;
typedef struct fp8bq_quant_job {
  int32_t kind;
  int32_t reserved; /* set to 0 */
  const void* x;
  int64_t rows;
  int64_t cols;
  int64_t ldx;
  void* q;
  void* scales;
  void* qt;
  void* scales_t;
} fp8bq_quant_job;
int fp8bq_quantize_group(const fp8bq_quant_job* jobs, int njobs, int fmt, fp8bq_stream_t stream);

/*
 * Blockwise-FP8 GEMM ("精度" section of the ModelScope post; "方法" of the
 * digest):  D[m, n] = sum over 128-blocks kb of  sA(m,kb) * sB(n,kb) *
 * sum_{k in kb} qA[m,k] * qB[n,k], accumulated in FP32 on the tensor cores,
 * rounded once to BF16 (round-to-nearest-even).
 *   forward  A = quantize_act(X), B = quantize_weight(W)        D = Y [M, N]
 *   dgrad    A = quantize_act(dY), B = W^T (k_major = 0)        D = dX [M, K_w]
 *   wgrad    A = quantize_act_t(dY), B = quantize_act_t(X)      D = dW [N, K]
 * FP32 scales run the per-128-K promotion path (partial products in tensor
 * memory, rescaled into FP32 accumulators); UE8M0 scales on both operands run
 * the block-scaled MMA (MXFP8 route); a mixed pair (one operand FP32, the
 * other UE8M0: DeepSeek-V3-style blocks meeting MXFP8 ones) runs the
 * promotion path with the UE8M0 scales decoded to 2^e.
 *   D       BF16 [M, N], leading dimension ldd (ldd >= N, ldd % 8 == 0); FP32
 *           with FP8BQ_GEMM_ACCUMULATE_F32.
 *   K       contraction length, K % 128 == 0, K > 0.
 *   flags   0, or FP8BQ_GEMM_ACCUMULATE_F32: D is then FP32 (ld ldd floats)
 *           and the product is added into it, D += A B^T, each element
 *           rounded once from D_old + the FP32 accumulator (the weight
 *           gradient added into an FP32 master gradient: "方法" keeps master
 *           weights and optimizer state in FP32).  Built for operands that are
 *           both row groups (1x128 or 1x32), k_major, E4M3; other
 *           combinations give ERR_UNSUPPORTED.  Other flag bits give
 *           ERR_INVALID_ARG.
 * Errors: ERR_INVALID_ARG, ERR_SHAPE (M,N <= 0, K % 128 != 0, N % 8 != 0),
 * ERR_ALIGN (a pointer not 16-B aligned, a leading dimension not a multiple
 * of 16 bytes), ERR_UNSUPPORTED (BF16 B, a BF16 A whose fmt differs from
 * B's, row-group B that is not k-major, MX operands mixed with other
 * granularities or not both k-major UE8M0), ERR_CUDA (tensor-map encoding or
 * launch failed).
 */
int fp8bq_gemm(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
               int64_t K, int64_t ldd, uint32_t flags, fp8bq_stream_t stream);

/*
 * fp8bq_gemm with a workspace that lets the kernel split tiles along K
 * (same product, same arguments and errors as fp8bq_gemm; the pages have no
 * counterpart: it is how the GEMM above fills a B200).  On C CTA pairs
 * (C = multiprocessors / 2) T output tiles of 256 x 256 take ceil(T / C)
 * rounds, the last one (T mod C) / C full; for the weight-gradient shapes of
 * the layer that round is mostly idle.  With a workspace, the tiles of that
 * round are shared along K by all C pairs, each pair taking one contiguous
 * run of their K blocks.  A tile's head piece (from K block 0) adds the FP32
 * partial sums that the tile's other pieces stored in their pairs' workspace
 * slots, in pair order, and rounds the tile to BF16 once: results are
 * bitwise reproducible, though not bitwise equal to fp8bq_gemm's (the same
 * FP32 sums, grouped differently).  The kernel splits only when there are
 * more tiles than CTA pairs and the split saves more than 5% of the launch.
 * Not used with FP8BQ_GEMM_ACCUMULATE_F32 (the workspace is then ignored).
 * The pieces of a tile wait for one another, so a split launch needs all its
 * CTA pairs resident at once (the GPU's SMs not held by other work); when
 * they cannot be, the waits expire after 2 s and fp8bq_check() reports
 * ERR_TIMEOUT.  Nothing is split when fewer than 4 K blocks per pair result.
 *   workspace        device memory of workspace_bytes, 256-byte aligned, all
 *                    zero before its first use; every call that completes
 *                    leaves its flags zero again.  After a call that fails on
 *                    the device (ERR_TIMEOUT), zero it before the next use.
 *                    Calls that may run at the same time need workspaces of
 *                    their own.  NULL: as fp8bq_gemm.
 *   workspace_bytes  at least fp8bq_gemm_workspace_bytes() (one 256 KB + 64
 *                    byte slot per CTA pair); a smaller workspace splits
 *                    nothing.
 * Errors: as fp8bq_gemm; ERR_INVALID_ARG for workspace_bytes < 0, ERR_ALIGN
 * for a workspace not 256-byte aligned.
 */
int fp8bq_gemm_ws(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N, int64_t K,
                  int64_t ldd, uint32_t flags, void* workspace, int64_t workspace_bytes, fp8bq_stream_t stream);

/* Workspace bytes for fp8bq_gemm_ws on the current device (one slot per CTA
 * pair), or -1 when no usable device is current. */
int64_t fp8bq_gemm_workspace_bytes(void);

/*
 * fp8bq_gemm_ws for callers that cannot allocate device memory: the
 * workspace is a fixed array inside this library instead of memory the
 * caller provides.  The pages have no counterpart; it exists for callers
 * that may not call cudaMalloc (it can synchronize the device, stalling
 * other streams), whose device memory is already held by another allocator,
 * or that are handed only their inputs and outputs, as plugin interfaces do.
 * Same arguments, product and errors as fp8bq_gemm, and the same tiles
 * split as fp8bq_gemm_ws with a workspace of fp8bq_gemm_workspace_bytes().
 *   Limit: the array has slots for 80 CTA pairs (20.98 MB, held on every GPU
 *   that loads the library until the process exits); on a device with more
 *   than 160 multiprocessors the call returns ERR_UNSUPPORTED.  Nothing is
 *   allocated: no cudaMalloc, no cudaFree.
 *   The first call in each CUDA context (on each device, and again after a
 *   cudaDeviceReset) looks up the array's device address with that device
 *   current (cudaGetSymbolAddress); make that first call before any stream
 *   capture.  Every call checks all its arguments first (an argument error
 *   queues nothing), then clears the array's flag words on the stream
 *   (cudaMemsetAsync) before the GEMM; with FP8BQ_GEMM_ACCUMULATE_F32,
 *   which splits nothing, the array is not touched.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents: calls that may overlap on the GPU (other streams, other host
 *   threads) race on it and must be ordered by the caller.
 */
int fp8bq_gemm_noalloc(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N, int64_t K,
                       int64_t ldd, uint32_t flags, fp8bq_stream_t stream);

/* Row stride of a 1x128-group scale array: rows rounded up to 128. */
int64_t fp8bq_row_scale_ld(int64_t rows);

/* Bytes of the scale array for an operand with `rows` rows and contraction
 * `contraction` (a multiple of 128); -1 on bad arguments (including
 * FP8BQ_GRAN_ROW_1x32 with FP32 scales). */
int64_t fp8bq_scales_bytes(int gran, int fmt, int64_t rows, int64_t contraction);

/*
 * Synchronizes `stream`, then reports the first device-side failure since the
 * last check: FP8BQ_ERR_TIMEOUT if a GEMM kernel's bounded wait expired (the
 * kernel then stopped early and its output is undefined), FP8BQ_ERR_CUDA if
 * the stream reported an error.  Clears the recorded state.
 */
int fp8bq_check(fp8bq_stream_t stream);

/*
 * Clock counters of the GEMM kernels, for measurement (the pages have no
 * counterpart).  GEMM launches on the current device issued after this call
 * add, for each of their CTAs, the SM cycles (clock64) and the nanoseconds
 * (globaltimer) between the CTA's start and its end to counters[0] and
 * counters[1]: counters[0] / counters[1] is then the SM clock, in GHz, that
 * the tensor cores ran at, which the driver's clock readings (sampled every
 * few milliseconds) do not resolve.  Costs two clock reads and two atomic
 * adds per CTA.
 *   counters  DEVICE memory of two uint64 (8-byte aligned), zeroed by the
 *             caller, or NULL to stop.  Launches already captured into a CUDA
 *             graph keep the pointer they were captured with.
 * Errors: ERR_ALIGN (counters not 8-byte aligned), ERR_UNSUPPORTED / ERR_CUDA
 * (no usable device).
 */
int fp8bq_set_clock_counters(unsigned long long* counters);

/* The cudaError_t value behind the last FP8BQ_ERR_CUDA of this thread. */
int fp8bq_last_cuda_error(void);

/* Static text for a status code. */
const char* fp8bq_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int fp8bq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BQ_H */
