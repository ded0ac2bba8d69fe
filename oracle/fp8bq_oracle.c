/*
 * fp8bq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU statement of what the blockwise-FP8
 * linear layer computes.  Only the test-suite, the smoke check and the
 * benchmark's cpu_baseline leg may load this file's library; the product path
 * (the CUDA library) never calls it and shares no code with it.
 *
 * What the method is (sources, by page title and section):
 *   - "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090"
 *     (agihunt paper digest), section "方法": Transformer linear layers run in
 *     blockwise FP8 from random init; activations are grouped by 128,
 *     weights use 128x128 blocks; on Blackwell the MXFP8 route is taken;
 *     master weights and optimizer state stay BF16/FP32.
 *   - same page, section "术语", entry "blockwise FP8": a scale per local
 *     block, so that one outlier cannot blow up a single per-tensor scale.
 *   - "清华开源 Puro-2B" (ModelScope community post), section
 *     "精度：FP8 分块量化与净效率收益": the matmuls of the main linear layers
 *     run on the FP8 path (fine-grained block quantization after DeepSeek-V3);
 *     numerically sensitive work and training state stay BF16/FP32.
 *
 * Readings where the pages are silent:
 *   - FP8 format: OCP E4M3FN (bias 7, max 448, no infinities, S.1111.111 NaN).
 *   - fp32 scale: s = fl32(amax / 448), s = 1 for an all-zero group;
 *     code q = E4M3_RNE_satfinite(fl32(x / s)).
 *   - power-of-two (UE8M0) scale, the MXFP8 reading of "MXFP8 on Blackwell":
 *     e = the smallest integer with amax <= 448 * 2^e, clamped to [-127,127],
 *     e = 0 for an all-zero group; stored byte e + 127; q = enc(x * 2^-e).
 *   - dequantized value: dec(q) * s; the GEMM is the plain product of the
 *     dequantized operands, evaluated in float64.
 *
 * Scale layouts (a library choice; the pages fix none):
 *   - 1x128 row groups of an operand with R rows and contraction length C:
 *     scales[cb * round_up(R,128) + r]; pad entries r >= R hold the neutral
 *     scale (1.0f, or byte 127).
 *   - 128x128 blocks: scales[cb * ceil(R/128) + rb].
 *   - 1x32 row groups (the other reading of "MXFP8 on Blackwell": the OCP
 *     Microscaling format's 32-element blocks with E8M0 scales): as 1x128
 *     row groups with 32 in place of 128, scales[cb32 * round_up(R,128) + r].
 *
 * Parity status: every function here is pinned by tests in tests/ (codec
 * against torch's float8_e4m3fn conversion and the closed-form grid,
 * quantizers against invariants and orientation identities, GEMM against a
 * numpy float64 product and an exact integer case).
 *
 * No SIMD, no blocking: loops follow the definition.  OpenMP only splits
 * independent groups or output rows across threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_SCALE_FP32 0
#define OR_SCALE_UE8M0 1
#define OR_GRAN_ROW 0
#define OR_GRAN_BLOCK 1
#define OR_GRAN_ROW32 2
#define OR_GROUP 128

/* ---------------------------------------------------------------- codec -- */

/* OCP 8-bit FP, E4M3FN: sign, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN; there is
 * no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_decode(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 15;
  int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(8.0 + (double)m, e - 10);
  return sign ? -v : v;
}

/* Round-to-nearest-even onto the E4M3 grid with saturation to +-448.
 * Precondition: f is not NaN (finite inputs are the method's contract);
 * +-Inf saturates like any value above 448.  The sign of zero is kept. */
uint8_t oracle_e4m3_encode(float f) {
  uint8_t sign = signbit(f) ? 0x80 : 0x00;
  double a = fabs((double)f);
  if (a >= 448.0) return sign | 0x7E;
  /* grid spacing: 2^-9 below 2^-5 (subnormals and the first binade share
   * it), 2^(E-3) in the binade [2^E, 2^(E+1)) above that. */
  int E;
  if (a < ldexp(1.0, -6)) {
    E = -6;
  } else {
    (void)frexp(a, &E);
    E -= 1;
  }
  double quantum = ldexp(1.0, E - 3);
  double n = nearbyint(a / quantum); /* exact quotient; default mode = RNE */
  double v = n * quantum;            /* may carry into the next binade */
  if (v == 0.0) return sign;
  int Ev;
  double fr = frexp(v, &Ev); /* v = fr * 2^Ev, fr in [0.5, 1) */
  Ev -= 1;                   /* v = (2 fr) * 2^Ev */
  if (Ev < -6) {
    /* subnormal: v = m * 2^-9 with m in 1..7 */
    int m = (int)(v / ldexp(1.0, -9));
    return sign | (uint8_t)m;
  }
  int m = (int)((2.0 * fr - 1.0) * 8.0);
  return sign | (uint8_t)(((Ev + 7) << 3) | m);
}

/* UE8M0 exponent: the smallest integer e with amax <= 448 * 2^e, found by an
 * exact search (448 * 2^e is representable), clamped to [-127, 127]. */
int oracle_ue8m0_exponent(float amax) {
  double a = (double)amax;
  if (a == 0.0) return 0;
  int e = 0;
  while (ldexp(448.0, e) < a) e++;
  while (e > -200 && ldexp(448.0, e - 1) >= a) e--;
  if (e > 127) e = 127;
  if (e < -127) e = -127;
  return e;
}

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------ group quantizer -- */

/* Quantize one group of n values (a 1x128 group or a 128x128 block).
 * Writes n codes and returns the scale through *s32 (fp32 format) or *e8
 * (UE8M0 byte).  Steps: amax -> scale -> codes, as in the file header. */
static void quantize_group(const float* v, int64_t n, int fmt, uint8_t* codes,
                           float* s32, uint8_t* e8) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; i++) {
    float a = fabsf(v[i]);
    if (a > amax) amax = a;
  }
  if (fmt == OR_SCALE_FP32) {
    float s = (amax == 0.0f) ? 1.0f : amax / 448.0f; /* IEEE single division */
    for (int64_t i = 0; i < n; i++) {
      float y = v[i] / s; /* IEEE single division */
      codes[i] = oracle_e4m3_encode(y);
    }
    *s32 = s;
  } else {
    int e = oracle_ue8m0_exponent(amax);
    for (int64_t i = 0; i < n; i++) {
      double y = ldexp((double)v[i], -e); /* exact scaling by 2^-e */
      codes[i] = oracle_e4m3_encode((float)y);
    }
    *e8 = (uint8_t)(e + 127);
  }
}

static int64_t round_up128(int64_t r) { return (r + 127) / 128 * 128; }

static void put_scale(void* scales, int fmt, int64_t idx, float s32, uint8_t e8) {
  if (fmt == OR_SCALE_FP32)
    ((float*)scales)[idx] = s32;
  else
    ((uint8_t*)scales)[idx] = e8;
}

/* Fill the pad entries r in [R, round_up(R,128)) of a row-group scale array. */
static void fill_row_pad(void* scales, int fmt, int64_t R, int64_t ncb) {
  int64_t ld = round_up128(R);
  for (int64_t cb = 0; cb < ncb; cb++)
    for (int64_t r = R; r < ld; r++) put_scale(scales, fmt, cb * ld + r, 1.0f, 127);
}

/* Groups of G (128, or 32 for MX blocks) along the columns of X [M, K] (K is
 * the contraction of the forward and dgrad GEMMs).  Output q [M, K] (ld K),
 * scales [K/G][round_up(M,128)].  Requires K % G == 0. */
int oracle_quantize_act_g(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                          uint8_t* q, void* scales, int fmt, int G) {
  if ((G != 128 && G != 32) || M < 0 || K < 0 || K % G != 0 || ldx < K) return -2;
  int64_t ncb = K / G;
  int64_t lds = round_up128(M);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < M; r++) {
    float v[OR_GROUP];
    uint8_t c[OR_GROUP];
    for (int64_t g = 0; g < ncb; g++) {
      for (int j = 0; j < G; j++) v[j] = bf16_to_f32(x[r * ldx + g * G + j]);
      float s32 = 0.0f;
      uint8_t e8 = 0;
      quantize_group(v, G, fmt, c, &s32, &e8);
      for (int j = 0; j < G; j++) q[r * K + g * G + j] = c[j];
      put_scale(scales, fmt, g * lds + r, s32, e8);
    }
  }
  fill_row_pad(scales, fmt, M, ncb);
  return 0;
}

int oracle_quantize_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                        uint8_t* q, void* scales, int fmt) {
  return oracle_quantize_act_g(x, M, K, ldx, q, scales, fmt, OR_GROUP);
}

/* Groups of G along the rows (tokens) of X [M, K], i.e. the act quantizer
 * applied to X^T, as the weight-gradient GEMM contracts over tokens.
 * Output qt [K, M] (ld M), scales [M/G][round_up(K,128)].
 * Requires M % 128 == 0. */
int oracle_quantize_act_t_g(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                            uint8_t* qt, void* scales, int fmt, int G) {
  if ((G != 128 && G != 32) || M < 0 || K < 0 || M % OR_GROUP != 0 || ldx < K) return -2;
  int64_t ncb = M / G;
  int64_t lds = round_up128(K);
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < K; c++) {
    float v[OR_GROUP];
    uint8_t cd[OR_GROUP];
    for (int64_t g = 0; g < ncb; g++) {
      for (int j = 0; j < G; j++) v[j] = bf16_to_f32(x[(g * G + j) * ldx + c]);
      float s32 = 0.0f;
      uint8_t e8 = 0;
      quantize_group(v, G, fmt, cd, &s32, &e8);
      for (int j = 0; j < G; j++) qt[c * M + g * G + j] = cd[j];
      put_scale(scales, fmt, g * lds + c, s32, e8);
    }
  }
  fill_row_pad(scales, fmt, K, ncb);
  return 0;
}

int oracle_quantize_act_t(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                          uint8_t* qt, void* scales, int fmt) {
  return oracle_quantize_act_t_g(x, M, K, ldx, qt, scales, fmt, OR_GROUP);
}

/* 128x128 blocks of W [N, K]; blocks at the row edge (N % 128 != 0) cover the
 * valid rows only.  Output q [N, K] (ld K), scales [K/128][ceil(N/128)].
 * Requires K % 128 == 0. */
int oracle_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                           uint8_t* q, void* scales, int fmt) {
  if (N < 0 || K < 0 || K % OR_GROUP != 0 || ldw < K) return -2;
  int64_t nkb = K / OR_GROUP;
  int64_t nnb = (N + OR_GROUP - 1) / OR_GROUP;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t nb = 0; nb < nnb; nb++) {
    for (int64_t kb = 0; kb < nkb; kb++) {
      float* v = (float*)malloc(sizeof(float) * OR_GROUP * OR_GROUP);
      uint8_t* cd = (uint8_t*)malloc(OR_GROUP * OR_GROUP);
      int64_t rows = N - nb * OR_GROUP;
      if (rows > OR_GROUP) rows = OR_GROUP;
      int64_t n = 0;
      for (int64_t i = 0; i < rows; i++)
        for (int j = 0; j < OR_GROUP; j++)
          v[n++] = bf16_to_f32(w[(nb * OR_GROUP + i) * ldw + kb * OR_GROUP + j]);
      float s32 = 0.0f;
      uint8_t e8 = 0;
      quantize_group(v, n, fmt, cd, &s32, &e8);
      n = 0;
      for (int64_t i = 0; i < rows; i++)
        for (int j = 0; j < OR_GROUP; j++) q[(nb * OR_GROUP + i) * K + kb * OR_GROUP + j] = cd[n++];
      put_scale(scales, fmt, kb * nnb + nb, s32, e8);
      free(v);
      free(cd);
    }
  }
  return 0;
}

/* ---------------------------------------------- SwiGLU (the producer op) -- */

/* Round a double to the nearest bfloat16, ties to even, in one step (no
 * intermediate float), keeping the sign of zero.  bf16 keeps 8 significant
 * bits with fp32's exponent range (subnormal quantum 2^-133). */
static uint16_t f64_to_bf16_rne(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e); /* a = m 2^e, m in [0.5, 1) */
  int E = e - 1;
  if (E < -126) E = -126;
  double quantum = ldexp(1.0, E - 7);
  double n = a / quantum; /* exact: power-of-two scaling */
  double fl = floor(n);
  double rem = n - fl;
  if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) == 1.0)) fl += 1.0;
  float f = (float)(fl * quantum); /* <= 9 significant bits: exact in float */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | (u >> 16));
}

/* The down projection's input: SwiGLU of the fused gate/up output.  gu is
 * BF16 [M, 2F] holding [gate | up] (the gate/up GEMM's two halves side by
 * side); h[r][c] = silu(g) * u with silu(g) = g / (1 + e^-g), g = gu[r][c],
 * u = gu[r][F + c], evaluated in float64 (h64, optional) and rounded once to
 * bfloat16 (h, ld F): the activation the layer stores in BF16 ("清华开源
 * Puro-2B", section "精度": activations outside the FP8 matmuls stay BF16). */
void oracle_swiglu(const uint16_t* gu, int64_t M, int64_t F, int64_t ld, uint16_t* h, double* h64) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < M; r++) {
    for (int64_t c = 0; c < F; c++) {
      double g = (double)bf16_to_f32(gu[r * ld + c]);
      double u = (double)bf16_to_f32(gu[r * ld + F + c]);
      double v = g / (1.0 + exp(-g)) * u;
      if (h64) h64[r * F + c] = v;
      h[r * F + c] = f64_to_bf16_rne(v);
    }
  }
}

/* The QKV and gate/up projections' input: RMSNorm of the block's input.
 * x is BF16 [M, K] (ld), gamma BF16 [K]; per row r the mean square
 * ms = sum_k x[r][k]^2 / K and rstd[r] = 1 / sqrt(ms + eps), then
 * h[r][k] = x[r][k] * rstd[r] * gamma[k], all in float64 (h64 and rstd64
 * optional), h rounded once to bfloat16 (ld K): the normalized activation
 * the layer keeps in BF16 ahead of the FP8 matmuls ("清华开源 Puro-2B",
 * section "精度"; a Qwen3-like block normalizes before QKV and gate/up). */
void oracle_rmsnorm(const uint16_t* x, int64_t M, int64_t K, int64_t ld, const uint16_t* gamma, double eps,
                    uint16_t* h, double* h64, double* rstd64) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < M; r++) {
    double ss = 0.0;
    for (int64_t k = 0; k < K; k++) {
      double v = (double)bf16_to_f32(x[r * ld + k]);
      ss += v * v;
    }
    double rs = 1.0 / sqrt(ss / (double)K + eps);
    if (rstd64) rstd64[r] = rs;
    for (int64_t k = 0; k < K; k++) {
      double v = (double)bf16_to_f32(x[r * ld + k]) * rs * (double)bf16_to_f32(gamma[k]);
      if (h64) h64[r * K + k] = v;
      h[r * K + k] = f64_to_bf16_rne(v);
    }
  }
}

/* ------------------------------------------------------------------ GEMM -- */

/* A quantized operand seen as a logical matrix [rows, C] with contraction C:
 *   element (r, k) is q[r*ld + k] when k_major, else q[k*ld + r];
 *   its scale is scales[(k/G)*s_stride_k + t*s_stride_r], where t = r for
 *   row groups and t = r/128 for 128x128 blocks, and G = 32 for 1x32 row
 *   groups, 128 otherwise. */
typedef struct {
  const uint8_t* q;
  int64_t ld;
  int32_t k_major;
  int32_t gran;
  const void* scales;
  int32_t fmt;
  int32_t pad_;
  int64_t s_stride_k;
  int64_t s_stride_r;
} oracle_operand;

static double dequant(const oracle_operand* op, int64_t r, int64_t k) {
  uint8_t c = op->k_major ? op->q[r * op->ld + k] : op->q[k * op->ld + r];
  int64_t t = (op->gran == OR_GRAN_BLOCK) ? r / OR_GROUP : r;
  int64_t g = (op->gran == OR_GRAN_ROW32) ? 32 : OR_GROUP;
  int64_t si = (k / g) * op->s_stride_k + t * op->s_stride_r;
  double s = (op->fmt == OR_SCALE_FP32) ? (double)((const float*)op->scales)[si]
                                        : ldexp(1.0, (int)((const uint8_t*)op->scales)[si] - 127);
  return oracle_e4m3_decode(c) * s;
}

/* D[i][j] = sum_k deq(A)[rows[i], k] * deq(B)[cols[j], k] in float64, for the
 * requested output rows and columns (all of them for small shapes; a seeded
 * sample of full rows and full columns at large ones). */
void oracle_gemm(const oracle_operand* A, const oracle_operand* B, int64_t C,
                 const int64_t* rows, int64_t nr, const int64_t* cols, int64_t nc,
                 double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nr; i++) {
    double* a = (double*)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    for (int64_t k = 0; k < C; k++) a[k] = dequant(A, rows[i], k);
    for (int64_t j = 0; j < nc; j++) {
      double acc = 0.0;
      for (int64_t k = 0; k < C; k++) acc += a[k] * dequant(B, cols[j], k);
      out[i * nc + j] = acc;
    }
    free(a);
  }
}

/* The weight gradient added into an FP32 master gradient (the digest's
 * "方法": master weights and optimizer state stay in FP32): out[i][j] =
 * d0[rows[i]][cols[j]] + the product above, in float64.  d0 is the FP32
 * gradient before the call, row-major with leading dimension ldd0. */
void oracle_gemm_accumulate(const oracle_operand* A, const oracle_operand* B, int64_t C,
                            const int64_t* rows, int64_t nr, const int64_t* cols, int64_t nc,
                            const float* d0, int64_t ldd0, double* out) {
  oracle_gemm(A, B, C, rows, nr, cols, nc, out);
  for (int64_t i = 0; i < nr; i++)
    for (int64_t j = 0; j < nc; j++) out[i * nc + j] += (double)d0[rows[i] * ldd0 + cols[j]];
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
