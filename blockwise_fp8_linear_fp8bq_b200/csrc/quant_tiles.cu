// quant_tiles.cu -- TMA-fed persistent quantizer for activations and output
// gradients ("Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within
// $5090", section "方法": activations quantized in groups of 128).
//
// One kernel template, three products of the same BF16 tile X[m0:m0+128,
// k0:k0+128]:
//   ROWS  1x128 groups along K: codes q [M, K] and scales [K/128][lds_m]
//         (the forward / dgrad A operand);
//   COLS  1x128 groups along the tokens M: codes qT [K, M] and scales
//         [M/128][lds_k] (the wgrad operands);
//   both  in one pass, reading X once (the backward pass needs both layouts
//         of dY, and the forward + wgrad both layouts of X).
//
// A persistent CTA per SM: one producer warp streams 128x128 tiles with TMA
// (two 64-column boxes, 128-byte swizzle) into a three-stage ring; sixteen
// consumer warps quantize out of shared memory and store codes and scales
// straight from registers.  Every wait is bounded (status word, as in the
// GEMM).
//
// The producer ops feed the same kernel: SwiGLU of a [gate | up] tile pair
// and RMSNorm of an X tile (with its row statistics from rstd_kernel), each
// warp computing the BF16 h of the rows it quantizes.  Their EXACT variants
// round h once from its exact value: FP32 where a proven error bound decides
// the BF16 rounding, float64 for the few values it leaves open.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace fp8bq {
namespace {

// Three 32 KB stages: measured in one process against 2, 4, 5, 6 and 7, three
// was the fastest over the layer's launches (the gate/up dY dual pass 136 µs
// against 150 µs with six; two starved the consumers): a deeper ring only
// puts more reads in flight against the codes being written.
constexpr int kQStages = 3;
constexpr int kQConsumers = 16;                 // consumer warps 0..15; warp 16 produces
constexpr int kQThreads = 32 * (kQConsumers + 1);
constexpr uint32_t kQBox = 128 * 128;           // 64 bf16 columns x 128 rows: 16 KB
constexpr uint32_t kQStage = 2 * kQBox;
// Shared-memory layout.  SW (SwiGLU producer fused in): a stage holds the
// gate tile and the up tile (64 KB), three stages, and an h-ready barrier
// per stage; otherwise one 32 KB tile a stage, kQStages stages.
template <bool SW>
struct QCfg {
  static constexpr int kStages = SW ? 3 : kQStages;
  static constexpr uint32_t kStage = SW ? 2 * kQStage : kQStage;
  static constexpr uint32_t kOffBar = kStages * kStage;
  static constexpr uint32_t kNumBars = 3 * kStages;  // full[S], empty[S], hready[S]
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // abort flag; then the grouped kernel's
  static constexpr uint32_t kRedBytes = kStages * kQConsumers * 4;  // per-stage weight-block amax partials
  static constexpr uint32_t kSmem = kOffMisc + 16 + kRedBytes + 2048;  // + slack for 2048-byte alignment
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr int kQTimeoutProducer = 11;
constexpr int kQTimeoutConsumer = 12;

struct QParams {
  CUtensorMap tmX;  // bf16 [M rows, K cols]; box 64 x 128; 128-byte swizzle
  int64_t M, K;
  uint8_t* q;       // ROWS: codes [M, K]
  void* s_rows;     //       scales [K/128][lds_m]
  int64_t lds_m;
  uint8_t* qt;      // COLS: codes [K, M]
  void* s_cols;     //       scales [M/128][lds_k]
  int64_t lds_k;
  int tiles_k, num_tiles;
  uint32_t tk_magic;  // floor((2^32 - 1) / tiles_k): tile index division without a divide
  int* status;
  uint64_t limit_ns;
  // SwiGLU producer: X is h = silu(gate) * up of tmX's [gate | up] columns
  int64_t up_off;   // column of up[0] (= F)
  uint16_t* h;      // optional BF16 h [M, K] (ld ldh) written on the way (SwiGLU or RMSNorm)
  int64_t ldh;
  // RMSNorm producer: X is h = x * rstd[row] * gamma[col]
  const float* rstd;       // [M]
  const double* rstd64;    // [M], the exact RMSNorm's float64 row statistic
  const uint16_t* gamma;   // BF16 [K]
};

// Tile t of a job -> (row block, column block) = (t / tiles_k, t % tiles_k):
// q = floor(t m / 2^32) with m = floor((2^32 - 1) / tiles_k) is the quotient
// or one less (t < 2^31), so one correction step gives the exact division.
__device__ __forceinline__ void tile_rc(const QParams& p, int t, int64_t& m0, int64_t& k0) {
  const uint32_t n = static_cast<uint32_t>(t);
  const uint32_t d = static_cast<uint32_t>(p.tiles_k);
  uint32_t q = __umulhi(n, p.tk_magic);
  uint32_t r = n - q * d;
  if (r >= d) {
    ++q;
    r -= d;
  }
  m0 = static_cast<int64_t>(q) * 128;
  k0 = static_cast<int64_t>(r) * 128;
}

// h = x * rstd * gamma in fp32 (two roundings), rounded to bf16 (nearest,
// ties to even): within one bf16 ulp of the exact product.  g is the pair's
// gamma, already in fp32.
__device__ __forceinline__ uint32_t rmsnorm_bf16x2(uint32_t x2, float2 rs2, float2 g) {
  const float2 h = __fmul2_rn(__fmul2_rn(make_float2(bf16_lo(x2), bf16_hi(x2)), rs2), g);
  return pack_bf16x2(h.x, h.y);
}

// True when an fp32 value whose error bound is `ulp` ulps cannot be rounded
// to bf16 with certainty: a rounding boundary (an fp32 whose low 16 bits are
// 0x8000) lies within `ulp` of it, or it lies outside [2^-100, 2^127), where
// its ulps stop being relative (or an intermediate may have overflowed).
__device__ __forceinline__ bool bf16_undecided(float h, uint32_t ulp) {
  const uint32_t mag = __float_as_uint(h) & 0x7FFFFFFFu;
  const bool near = ((mag + (ulp - 0x8000u)) & 0xFFFFu) <= 2 * ulp;
  const bool range = (mag - 0x0D800000u) >= (0x7F000000u - 0x0D800000u);
  return near || range;
}

// h = silu(g) u = g u / (1 + e^-g) for one value the fast path left
// undecided, rounded once to bf16 (nearest, ties to even).  First in fp32
// with the accurate exponential (within 2 ulp, the documented bound of
// expf), the add (half an ulp) and the IEEE division (half an ulp): within
// 2 (2 + 0.5 + 0.5) = 6 ulp of h for |g| <= 80; if that still leaves the
// rounding open, in float64 in the order of the definition,
// (g / (1 + e^-g)) u, rounded once from there.  Out of line: it runs for a
// few values in a thousand.
static __device__ __noinline__ uint32_t swiglu_slow_bf16(float g, float u) {
  if (fabsf(g) <= 80.0f) {
    const float h = __fdiv_rn(g * u, 1.0f + expf(-g));
    if (!bf16_undecided(h, 8)) return pack_bf16x2(h, 0.0f) & 0xFFFFu;
  }
  const double gd = g;
  const double v = gd / (1.0 + exp(-gd)) * static_cast<double>(u);
  uint16_t r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(v));
  return r;
}

// Ulps of the fast path's error bound (rounded up) and the gate magnitude
// up to which it holds.
constexpr uint32_t kSwiBoundUlp = 64;
constexpr float kSwiGateMax = 16.0f;

// h = silu(g) u = g u / (1 + e^-g) for two bf16 pairs, from the fp32 value
// hf = g u / (1 + e^-g) with the fast exponential and division.
//
// Default (EXACT false): hf rounded to bf16 (nearest, ties to even; finite
// values), within one bf16 ulp of the exact value: hf is within a few parts
// in 2^20 of it, and the bf16 rounding hides that except next to a rounding
// boundary.  For gate < -87, e^-g overflows and h = +-0.
//
// EXACT: each value rounded once to bf16 from the exact one.  g u is exact
// (two 8-bit significands); the exponential is within 2 + floor(1.173 |g|)
// ulp (the documented bound of __expf), the add within half an ulp, the
// division within 2 ulp (__fdividef, divisor below 2^126), so hf is within
// 2 (2 + 1.173 |g| + 2.5) < 48 ulp of h for |g| <= 16.  Its bf16 rounding is
// h's unless bf16_undecided says otherwise; those values and |g| > 16 take
// swiglu_slow_bf16.
template <bool EXACT>
__device__ __forceinline__ uint32_t swiglu_bf16x2(uint32_t g2, uint32_t u2) {
  float g[2], u[2], h[2];
  bool slow[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    g[k] = k ? bf16_hi(g2) : bf16_lo(g2);
    u[k] = k ? bf16_hi(u2) : bf16_lo(u2);
    h[k] = __fdividef(g[k] * u[k], 1.0f + __expf(-g[k]));
    if constexpr (EXACT) slow[k] = bf16_undecided(h[k], kSwiBoundUlp) || !(fabsf(g[k]) <= kSwiGateMax);
  }
  uint32_t r = pack_bf16x2(h[0], h[1]);  // round to nearest even
  if constexpr (EXACT) {
    if (slow[0]) r = (r & 0xFFFF0000u) | swiglu_slow_bf16(g[0], u[0]);
    if (slow[1]) r = (r & 0x0000FFFFu) | (swiglu_slow_bf16(g[1], u[1]) << 16);
  }
  return r;
}

// RMSNorm rounded once from the exact value h = x rstd gamma, given rstd in
// float64 (rs64) and rs = its fp32 rounding.  With rs, t = x rs and hf =
// t gamma all normal fp32 values, hf is within 2^-24 (rs) + 2 x 2^-24 (the
// two products' roundings) of h, relative, i.e. within 3 ulp (plus the
// float64 rstd's own error, below 2^-33 for any K): its bf16 rounding is h's
// unless bf16_undecided(hf, 8) says otherwise.  Those values, and the values
// of a row whose rs is not a normal fp32 (row_slow) or whose t is not one,
// are evaluated in float64 in the definition's order, (x rstd) gamma, and
// rounded once.
constexpr uint32_t kNormBoundUlp = 8;

static __device__ __noinline__ uint32_t rmsnorm_f64_bf16(float x, double rs64, float g) {
  const double v = static_cast<double>(x) * rs64 * static_cast<double>(g);
  uint16_t r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(v));
  return r;
}

// |v| outside [2^-126, 2^127): not a normal fp32 (or near overflow).
__device__ __forceinline__ bool f32_not_normal(float v) {
  const uint32_t mag = __float_as_uint(v) & 0x7FFFFFFFu;
  return (mag - 0x00800000u) >= (0x7F000000u - 0x00800000u);
}

__device__ __forceinline__ uint32_t rmsnorm_exact_bf16x2(uint32_t x2, float2 rs2, float2 g, double rs64,
                                                         bool row_slow) {
  const float2 xx = make_float2(bf16_lo(x2), bf16_hi(x2));
  const float2 t = __fmul2_rn(xx, rs2);
  const float2 h = __fmul2_rn(t, g);
  uint32_t r = pack_bf16x2(h.x, h.y);
  if (row_slow || f32_not_normal(t.x) || bf16_undecided(h.x, kNormBoundUlp))
    r = (r & 0xFFFF0000u) | rmsnorm_f64_bf16(xx.x, rs64, g.x);
  if (row_slow || f32_not_normal(t.y) || bf16_undecided(h.y, kNormBoundUlp))
    r = (r & 0x0000FFFFu) | (rmsnorm_f64_bf16(xx.y, rs64, g.y) << 16);
  return r;
}

// Byte offset of 16-byte chunk c (0..15, 8 bf16 each) of tile row r: chunks
// 0..7 in the first box, 8..15 in the second; 128-byte swizzle within a box.
__device__ __forceinline__ uint32_t tile_chunk(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kQBox + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Row groups: warp w, half-warp h, lane l16 own rows 8 w + 2 i + h (i < 4),
// chunk l16 (8 values); the amax is a 16-lane reduction.
template <int FMT, int G>
__device__ __forceinline__ void tile_rows_regs(const QParams& p, const uint4 (&v)[4], int64_t m0, int64_t k0,
                                               int warp, int lane) {
  const int half = lane >> 4;
  const int l16 = lane & 15;
  float m[4];
  uint32_t p2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // packed |max| of the 8 values (even columns in the low half, odd ones in the high)
    p2[i] = absmax_bf16x2(absmax_bf16x2(v[i].x, v[i].y), absmax_bf16x2(v[i].z, v[i].w));
  }
  // two rows per word (row 2j in the low half, 2j + 1 in the high one), so
  // one shuffle tree over the G / 8 lanes of the groups serves both rows
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t w = absmax_bf16x2(__byte_perm(p2[2 * j], p2[2 * j + 1], 0x5410),
                               __byte_perm(p2[2 * j], p2[2 * j + 1], 0x7632));
#pragma unroll
    for (int o = G / 16; o >= 1; o >>= 1) w = absmax_bf16x2(w, __shfl_xor_sync(0xffffffffu, w, o));
    w &= 0x7FFF7FFFu;
    m[2 * j] = bf16_lo(w);
    m[2 * j + 1] = bf16_hi(w);
  }
  static_assert(FMT == kFmtUe8m0 || G == 128, "FP32 scales come in 1x128 groups");
  GroupScale gs[4];
  GroupScale own{};  // UE8M0: the scale of row slot l16 mod 4
  if constexpr (FMT == kFmtFp32 && G == 128) {
    // one scale per group, computed by lane 2 i + h and fetched by the others
    float mine = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float mi = __shfl_sync(0xffffffffu, m[i], (lane & 1) * 16);
      if ((lane >> 1) == i) mine = mi;
    }
    const GroupScale gmine = make_scale<FMT>(mine);
#pragma unroll
    for (int i = 0; i < 4; ++i) gs[i] = fetch_scale<FMT>(gmine, 2 * i + half);
  } else {
    // the G / 8 lanes of a group hold the same four row maxima: lane slot i
    // (i = l16 mod 4) computes row slot i's scale, and every lane fetches the
    // four multipliers from slots 0..3 of its group (one shuffle each, in
    // place of three scale computations)
    const int slot = l16 & 3;
    const float mine = slot == 0 ? m[0] : slot == 1 ? m[1] : slot == 2 ? m[2] : m[3];
    own = make_scale<FMT>(mine);
    const int first = lane & ~(G / 8 - 1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      gs[i] = own;
      gs[i].mul = __shfl_sync(0xffffffffu, own.mul, first + i);
    }
  }
  uint2 c[4];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = quant8_fast<FMT>(v[i], gs[i], slow);
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = quant8_exact<FMT>(v[i], gs[i]);
  }
  const int64_t r0 = m0 + 8 * warp + half;
  uint8_t* qrow = p.q + r0 * p.K + k0 + 8 * l16;
  const int64_t sg = k0 / G + (l16 * 8) / G;  // scales [K/G][lds_m]
  if constexpr (FMT == kFmtFp32) {
    // the first lane of each group stores its four rows' scales
    const bool lead = (l16 & (G / 8 - 1)) == 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t r = r0 + 2 * i;
      if (r < p.M) {
        *reinterpret_cast<uint2*>(qrow + 2 * i * p.K) = c[i];
        if (lead) store_scale<FMT>(p.s_rows, sg * p.lds_m + r, gs[i]);
      } else if (r < p.lds_m && lead) {
        store_neutral_scale<FMT>(p.s_rows, sg * p.lds_m + r);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (r0 + 2 * i < p.M) *reinterpret_cast<uint2*>(qrow + 2 * i * p.K) = c[i];
    }
    // lane slot i of each group (i < 4) stores row slot i's scale, its own
    const int gl = l16 & (G / 8 - 1);
    if (gl < 4) {
      const int64_t r = r0 + 2 * gl;
      if (r < p.M)
        store_scale<FMT>(p.s_rows, sg * p.lds_m + r, own);
      else if (r < p.lds_m)
        store_neutral_scale<FMT>(p.s_rows, sg * p.lds_m + r);
    }
  }
}

// The same, loading the warp's rows (8 warp + 2 i + half, chunk l16) from
// the staged tile.
template <int FMT, int G>
__device__ __forceinline__ void tile_rows(const QParams& p, uint32_t base, int64_t m0, int64_t k0, int warp,
                                          int lane) {
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = ld_shared_v4(base + tile_chunk(8 * warp + 2 * i + (lane >> 4), lane & 15));
  tile_rows_regs<FMT, G>(p, v, m0, k0, warp, lane);
}

// Byte i of r moves to byte i ^ j, for 0 <= j < 8: one byte permute per
// output word, taking the bytes of its own word (j < 4) or of its pair
// partner (j >= 4), each at byte index ^ (j & 3).
__device__ __forceinline__ uint32_t xor_bytes_selector(int j) {
  return (0x3210u ^ (static_cast<uint32_t>(j & 3) * 0x1111u)) | ((j & 4) ? 0x4444u : 0u);
}
__device__ __forceinline__ uint4 xor_bytes(const uint4& r, uint32_t sel) {
  return make_uint4(__byte_perm(r.x, r.y, sel), __byte_perm(r.y, r.x, sel), __byte_perm(r.z, r.w, sel),
                    __byte_perm(r.w, r.z, sel));
}

// Token groups: warp w takes box w & 1 and its column pairs 4 (w >> 1) ..
// + 3; lane (a = lane >> 3, j = lane & 7) owns pair a (two columns, one
// 32-bit word per token) and tokens 16 j .. 16 j + 15, so a column's 128
// tokens sit in the eight lanes of its pair and the amax is a shuffle
// reduction.  Load i of lane j reads token 16 j + (i ^ j): the eight lanes of
// a pair then read eight different swizzle phases and the warp's 32 reads
// hit 32 banks, and with the stage 2048-byte aligned every address is the
// lane's base XOR a constant.  The codes come out in that order and are
// permuted back (byte i to byte i ^ j) before each lane stores its 16
// consecutive tokens (8 lanes: one 128-byte row segment of the transposed
// codes).
template <int FMT, int G>
__device__ __forceinline__ void tile_cols(const QParams& p, uint32_t base, int64_t m0, int64_t k0, int warp,
                                          int lane) {
  const int box = warp & 1;
  const int a = lane >> 3;
  const int j = lane & 7;
  const int chunk = warp >> 1;  // 16-byte chunk holding the warp's 4 pairs
  // token r = 16 j + (i ^ j) sits at cbase + 128 r + 16 (chunk ^ (r & 7));
  // bits 4-10 of cbase + 2048 j are zero, so that is lbase ^ (128 i + 16 (i & 7))
  const uint32_t jj = static_cast<uint32_t>(j);
  const uint32_t lbase = (base + box * kQBox + 4 * a + 2048u * jj) ^ ((jj << 7) | (jj << 4)) ^
                         (static_cast<uint32_t>(chunk) << 4);
  uint32_t w[16];  // w[i]: token 16 j + (i ^ j)
  // bit 10 of lbase is clear (the stage is 2048-byte aligned and the other
  // terms sit in bits 2-9 and 11 up), so for loads 8-15 the XOR with 1024 is
  // an addition the load's immediate offset absorbs
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = lbase ^ static_cast<uint32_t>((i << 7) | (i << 4));
    w[i] = ld_shared_u32(a);
    w[i + 8] = ld_shared_u32(a + 1024u);
  }
  // packed |max| over the 16 tokens (both columns at once), then over the
  // 8 lanes of the pair
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) m2 = absmax_bf16x2(m2, w[i]);
#pragma unroll
  for (int o = G / 32; o >= 1; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  m2 &= 0x7FFF7FFFu;
  const float m0v = bf16_lo(m2), m1v = bf16_hi(m2);
  GroupScale s0, s1;
  GroupScale own{};  // UE8M0: the scale of column j mod 2 of the pair
  if constexpr (FMT == kFmtFp32 && G == 128) {
    // eight groups per warp: lane 2 a' + b computes column b of pair a'
    float mine = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float t0 = __shfl_sync(0xffffffffu, m0v, 8 * q);
      const float t1 = __shfl_sync(0xffffffffu, m1v, 8 * q);
      if (lane == 2 * q) mine = t0;
      if (lane == 2 * q + 1) mine = t1;
    }
    const GroupScale gmine = make_scale<FMT>(mine);
    s0 = fetch_scale<FMT>(gmine, 2 * a);
    s1 = fetch_scale<FMT>(gmine, 2 * a + 1);
  } else {
    // the G / 16 lanes of a token group hold the same two column maxima: an
    // even lane computes the first column's scale, an odd one the second's,
    // and each lane fetches both multipliers from its lane pair
    own = make_scale<FMT>((j & 1) ? m1v : m0v);
    s0 = own;
    s1 = own;
    s0.mul = __shfl_sync(0xffffffffu, own.mul, lane & ~1);
    s1.mul = __shfl_sync(0xffffffffu, own.mul, lane | 1);
  }
  // codes straight from the token words: the first column is the low bf16
  // of each word, the second the high one; two tokens per conversion
  uint2 ca[2], cb[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t c0[4], c1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = w[8 * h + 2 * k], hi = w[8 * h + 2 * k + 1];
      c0[k] = quant2_fast<FMT>(make_float2(bf16_lo(lo), bf16_lo(hi)), s0);
      c1[k] = quant2_fast<FMT>(make_float2(bf16_hi(lo), bf16_hi(hi)), s1);
    }
    ca[h] = make_uint2(c0[0] | (c0[1] << 16), c0[2] | (c0[3] << 16));
    cb[h] = make_uint2(c1[0] | (c1[1] << 16), c1[2] | (c1[3] << 16));
  }
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, s0.r == 0.0f || s1.r == 0.0f)) {
    // groups of tiny scale: the IEEE division on the columns split out
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 wa = make_uint4(__byte_perm(w[8 * h + 0], w[8 * h + 1], 0x5410),
                                  __byte_perm(w[8 * h + 2], w[8 * h + 3], 0x5410),
                                  __byte_perm(w[8 * h + 4], w[8 * h + 5], 0x5410),
                                  __byte_perm(w[8 * h + 6], w[8 * h + 7], 0x5410));
      const uint4 wb = make_uint4(__byte_perm(w[8 * h + 0], w[8 * h + 1], 0x7632),
                                  __byte_perm(w[8 * h + 2], w[8 * h + 3], 0x7632),
                                  __byte_perm(w[8 * h + 4], w[8 * h + 5], 0x7632),
                                  __byte_perm(w[8 * h + 6], w[8 * h + 7], 0x7632));
      ca[h] = quant8_exact<FMT>(wa, s0);
      cb[h] = quant8_exact<FMT>(wb, s1);
    }
  }
  const uint32_t xsel = xor_bytes_selector(j);
  const uint4 va = xor_bytes(make_uint4(ca[0].x, ca[0].y, ca[1].x, ca[1].y), xsel);
  const uint4 vb = xor_bytes(make_uint4(cb[0].x, cb[0].y, cb[1].x, cb[1].y), xsel);
  const int64_t c = k0 + 64 * box + 2 * (4 * chunk + a);
  const int64_t tok = m0 + 16 * j;
  const int64_t sidx = (m0 / G + (16 * j) / G) * p.lds_k + c;  // scales [M/G][lds_k]
  if constexpr (FMT == kFmtFp32) {
    // the first lane of each token group stores its two scales
    const bool lead = (j & (G / 16 - 1)) == 0;
    if (c < p.K) {
      *reinterpret_cast<uint4*>(p.qt + c * p.M + tok) = va;
      if (lead) store_scale<FMT>(p.s_cols, sidx, s0);
    } else if (c < p.lds_k && lead) {
      store_neutral_scale<FMT>(p.s_cols, sidx);
    }
    if (c + 1 < p.K) {
      *reinterpret_cast<uint4*>(p.qt + (c + 1) * p.M + tok) = vb;
      if (lead) store_scale<FMT>(p.s_cols, sidx + 1, s1);
    } else if (c + 1 < p.lds_k && lead) {
      store_neutral_scale<FMT>(p.s_cols, sidx + 1);
    }
  } else {
    if (c < p.K) *reinterpret_cast<uint4*>(p.qt + c * p.M + tok) = va;
    if (c + 1 < p.K) *reinterpret_cast<uint4*>(p.qt + (c + 1) * p.M + tok) = vb;
    // the first two lanes of each token group store the scales of the first
    // and the second column, each its own
    const int gl = j & (G / 16 - 1);
    if (gl < 2) {
      if (c + gl < p.K)
        store_scale<FMT>(p.s_cols, sidx + gl, own);
      else if (c + gl < p.lds_k)
        store_neutral_scale<FMT>(p.s_cols, sidx + gl);
    }
  }
}

// One 128x128 weight block (the tile itself): the amax over the whole tile
// (each warp's share as in tile_rows, then the 16 warps' partials through
// `red` and a named barrier of the consumer warps), one scale, and the codes
// of the tile's rows.  The block scale lands at (k0/128) * lds_m + m0/128,
// lds_m being ceil(N/128) for a weight [N, K].
template <int FMT>
__device__ __forceinline__ void tile_block(const QParams& p, uint32_t base, int64_t m0, int64_t k0, int warp, int lane,
                                           float* red) {
  const int half = lane >> 4;
  const int l16 = lane & 15;
  uint4 v[4];
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = ld_shared_v4(base + tile_chunk(8 * warp + 2 * i + half, l16));
    m2 = absmax_bf16x2(m2, absmax_bf16x2(absmax_bf16x2(v[i].x, v[i].y), absmax_bf16x2(v[i].z, v[i].w)));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  m2 &= 0x7FFF7FFFu;
  if (lane == 0) red[warp] = fmaxf(bf16_lo(m2), bf16_hi(m2));
  named_bar_sync(1, 32 * kQConsumers);
  float bm = red[0];
#pragma unroll
  for (int w = 1; w < kQConsumers; ++w) bm = fmaxf(bm, red[w]);
  const GroupScale gs = make_scale<FMT>(bm);
  uint2 c[4];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = quant8_fast<FMT>(v[i], gs, slow);
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = quant8_exact<FMT>(v[i], gs);
  }
  const int64_t r0 = m0 + 8 * warp + half;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + 2 * i;
    if (r < p.M) *reinterpret_cast<uint2*>(p.q + r * p.K + k0 + 8 * l16) = c[i];
  }
  if (warp == 0 && lane == 0) store_scale<FMT>(p.s_rows, (k0 / 128) * p.lds_m + m0 / 128, gs);
}

template <int FMT, bool ROWS, bool COLS, int G, bool SW, bool NORM, bool EXACT>
__global__ void __launch_bounds__(kQThreads, 1) quant_tile_kernel(const __grid_constant__ QParams p) {
  static_assert(G == 128 || (G == 32 && FMT == kFmtUe8m0), "1x32 groups use UE8M0 scales");
  using C = QCfg<SW>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  // stages 2048-byte aligned: a token-group lane's row addresses then differ
  // from one another only in bits 4-10 (see tile_cols)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 2047) &
                                             ~static_cast<uintptr_t>(2047));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto hready_bar = [&](int s) { return smem_u32(&bars[2 * S + s]); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  const WaitGuard guard{abort_flag, p.status, p.limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kQConsumers);
      mbar_init(hready_bar(s), kQConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kQConsumers) {
    // ------------------------------------------------------------ producer
    prefetch_tensormap(&p.tmX);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(empty_bar(s), ph ^ 1, guard, kQTimeoutProducer))) { ok = false; break; }
      if (elect_one()) {
        int64_t m0l, k0l;
        tile_rc(p, tile, m0l, k0l);
        const int32_t m0 = static_cast<int32_t>(m0l), k0 = static_cast<int32_t>(k0l);
        const uint32_t dst = smem_u32(smem + s * C::kStage);
        if (SW) {
          // gate columns k0 .. k0 + 127 and up columns F + k0 .. (F % 128 == 0)
          const int32_t u0 = static_cast<int32_t>(p.up_off) + k0;
          mbar_arrive_expect_tx(full_bar(s), 2 * kQStage);
          tma_load_2d(dst, &p.tmX, full_bar(s), k0, m0);
          tma_load_2d(dst + kQBox, &p.tmX, full_bar(s), k0 + 64, m0);
          tma_load_2d(dst + kQStage, &p.tmX, full_bar(s), u0, m0);
          tma_load_2d(dst + kQStage + kQBox, &p.tmX, full_bar(s), u0 + 64, m0);
        } else {
          // a box wholly past K (ragged K, COLS only) is not loaded: its
          // columns are never stored and form groups of their own
          const bool second = k0 + 64 < p.K;
          mbar_arrive_expect_tx(full_bar(s), second ? kQStage : kQBox);
          tma_load_2d(dst, &p.tmX, full_bar(s), k0, m0);
          if (second) tma_load_2d(dst + kQBox, &p.tmX, full_bar(s), k0 + 64, m0);
        }
      }
      __syncwarp();
    }
    // teardown: every load issued has landed before the CTA exits
    const uint32_t total = it;
    for (uint32_t j = (total > S ? total - S : 0); j < total; ++j)
      mbar_wait(full_bar(j % S), (j / S) & 1, guard, kQTimeoutProducer);
  } else {
    // ------------------------------------------------------------ consumers
    // RMSNorm: gamma of this thread's 8 columns and rstd of its 4 rows, for
    // the tile at hand (loaded one tile ahead, off the critical path)
    uint4 ng = make_uint4(0, 0, 0, 0);
    float nrs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    double nrs64[4] = {0.0, 0.0, 0.0, 0.0};  // exact RMSNorm: rstd in float64
    auto norm_load = [&](int tile) {
      if (tile >= p.num_tiles) return;
      int64_t tm0, tk0;
      tile_rc(p, tile, tm0, tk0);
      ng = __ldg(reinterpret_cast<const uint4*>(p.gamma + tk0 + 8 * (threadIdx.x % 16)));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t r = tm0 + 8 * warp + 2 * i + (lane >> 4);
        if constexpr (EXACT) {
          nrs64[i] = r < p.M ? __ldg(p.rstd64 + r) : 0.0;
          nrs[i] = __double2float_rn(nrs64[i]);
        } else {
          nrs[i] = r < p.M ? __ldg(p.rstd + r) : 0.0f;
        }
      }
    };
    if constexpr (NORM) norm_load(blockIdx.x);
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kQTimeoutConsumer))) break;
      int64_t m0, k0;
      tile_rc(p, tile, m0, k0);
      const uint32_t base = smem_u32(smem + s * C::kStage);
      // Producer ops (SwiGLU, RMSNorm): warp w computes h for the rows it
      // quantizes in 1x128 groups (8 w + 2 i + half, chunk l16), stores h in
      // place of the input tile and quantizes those rows from registers; the
      // token-group phase, which reads every row, waits for all warps' h.
      bool rows_done = false;
      if constexpr (SW || NORM) {
        const int half = lane >> 4, l16 = lane & 15;
        uint4 hv[4];
        float2 g0, g1, g2, g3;
        float rsv[4];
        double rsv64[4];
        if constexpr (NORM) {
          g0 = make_float2(bf16_lo(ng.x), bf16_hi(ng.x));
          g1 = make_float2(bf16_lo(ng.y), bf16_hi(ng.y));
          g2 = make_float2(bf16_lo(ng.z), bf16_hi(ng.z));
          g3 = make_float2(bf16_lo(ng.w), bf16_hi(ng.w));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            rsv[i] = nrs[i];
            rsv64[i] = nrs64[i];
          }
          norm_load(tile + gridDim.x);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 8 * warp + 2 * i + half;
          const uint32_t off = tile_chunk(r, l16);
          if constexpr (SW) {
            const uint4 g = ld_shared_v4(base + off);
            const uint4 u = ld_shared_v4(base + kQStage + off);
            hv[i] = make_uint4(swiglu_bf16x2<EXACT>(g.x, u.x), swiglu_bf16x2<EXACT>(g.y, u.y),
                               swiglu_bf16x2<EXACT>(g.z, u.z), swiglu_bf16x2<EXACT>(g.w, u.w));
          } else {
            const float2 rs2 = make_float2(rsv[i], rsv[i]);
            const uint4 x = ld_shared_v4(base + off);
            if constexpr (EXACT) {
              const bool row_slow = f32_not_normal(rsv[i]);
              hv[i] = make_uint4(rmsnorm_exact_bf16x2(x.x, rs2, g0, rsv64[i], row_slow),
                                 rmsnorm_exact_bf16x2(x.y, rs2, g1, rsv64[i], row_slow),
                                 rmsnorm_exact_bf16x2(x.z, rs2, g2, rsv64[i], row_slow),
                                 rmsnorm_exact_bf16x2(x.w, rs2, g3, rsv64[i], row_slow));
            } else
              hv[i] = make_uint4(rmsnorm_bf16x2(x.x, rs2, g0), rmsnorm_bf16x2(x.y, rs2, g1),
                                 rmsnorm_bf16x2(x.z, rs2, g2), rmsnorm_bf16x2(x.w, rs2, g3));
          }
          st_shared_v4(base + off, hv[i].x, hv[i].y, hv[i].z, hv[i].w);
          if (p.h != nullptr && m0 + r < p.M)
            *reinterpret_cast<uint4*>(p.h + (m0 + r) * p.ldh + k0 + 8 * l16) = hv[i];
        }
        if (ROWS) tile_rows_regs<FMT, G>(p, hv, m0, k0, warp, lane);
        rows_done = true;
        __syncwarp();
        if (lane == 0) mbar_arrive(hready_bar(s));
        if (!__all_sync(0xffffffffu, mbar_wait(hready_bar(s), ph, guard, kQTimeoutConsumer))) break;
      }
      if (ROWS && !rows_done) tile_rows<FMT, G>(p, base, m0, k0, warp, lane);
      if (COLS) tile_cols<FMT, G>(p, base, m0, k0, warp, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
  }
}

// ------------------------------------------------------- grouped launch --
// Several quantizations in one persistent launch: the tiles of job 0, then
// job 1, ... are one index space that the CTAs stride through, so the small
// tensors of a layer (a weight and an activation, say) share one pipeline
// ramp and one tail instead of paying one each.  A job is a row-group,
// token-group or dual activation quantization, or a 128x128 weight-block one.
constexpr int kQMaxJobs = 8;
constexpr int kQModeRows = 1, kQModeCols = 2, kQModeBlock = 4;  // rows | cols: both layouts

struct QGroup {
  QParams job[kQMaxJobs];
  int tile_end[kQMaxJobs];  // exclusive prefix sums of the jobs' tile counts
  int mode[kQMaxJobs];
  int njobs;
  int num_tiles;
  int* status;
  uint64_t limit_ns;
};

__device__ __forceinline__ int job_of(const QGroup& g, int tile, int& local) {
  int j = 0;
  while (j + 1 < g.njobs && tile >= g.tile_end[j]) ++j;
  local = tile - (j > 0 ? g.tile_end[j - 1] : 0);
  return j;
}

template <int FMT>
__global__ void __launch_bounds__(kQThreads, 1) quant_group_kernel(const __grid_constant__ QGroup g) {
  using C = QCfg<false>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 2047) &
                                             ~static_cast<uintptr_t>(2047));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  float* red_all = reinterpret_cast<float*>(smem + C::kOffMisc + 16);  // [S][kQConsumers] block partials
  const WaitGuard guard{abort_flag, g.status, g.limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kQConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kQConsumers) {
    // ------------------------------------------------------------ producer
    for (int j = 0; j < g.njobs; ++j) prefetch_tensormap(&g.job[j].tmX);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(empty_bar(s), ph ^ 1, guard, kQTimeoutProducer))) { ok = false; break; }
      if (elect_one()) {
        int lt = 0;
        const QParams& p = g.job[job_of(g, tile, lt)];
        int64_t m0l, k0l;
        tile_rc(p, lt, m0l, k0l);
        const int32_t m0 = static_cast<int32_t>(m0l), k0 = static_cast<int32_t>(k0l);
        const uint32_t dst = smem_u32(smem + s * C::kStage);
        // a box wholly past K (ragged K, token groups only) is not loaded
        const bool second = k0 + 64 < p.K;
        mbar_arrive_expect_tx(full_bar(s), second ? kQStage : kQBox);
        tma_load_2d(dst, &p.tmX, full_bar(s), k0, m0);
        if (second) tma_load_2d(dst + kQBox, &p.tmX, full_bar(s), k0 + 64, m0);
      }
      __syncwarp();
    }
    const uint32_t total = it;
    for (uint32_t j = (total > S ? total - S : 0); j < total; ++j)
      mbar_wait(full_bar(j % S), (j / S) & 1, guard, kQTimeoutProducer);
  } else {
    // ------------------------------------------------------------ consumers
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kQTimeoutConsumer))) break;
      int lt = 0;
      const int j = job_of(g, tile, lt);
      const QParams& p = g.job[j];
      const int mode = g.mode[j];
      int64_t m0, k0;
      tile_rc(p, lt, m0, k0);
      const uint32_t base = smem_u32(smem + s * C::kStage);
      if (mode == kQModeBlock) {
        tile_block<FMT>(p, base, m0, k0, warp, lane, red_all + s * kQConsumers);
      } else {
        if (mode & kQModeRows) tile_rows<FMT, 128>(p, base, m0, k0, warp, lane);
        if (mode & kQModeCols) tile_cols<FMT, 128>(p, base, m0, k0, warp, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
  }
}

// 2-D tensor map over bf16 X [rows, cols] (row pitch in bytes); 64 x 128 boxes,
// 128-byte swizzle; out-of-range elements read as zero.
bool encode_x(CUtensorMap* map, const void* x, int64_t rows, int64_t cols, int64_t ldx) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldx) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int FMT, bool ROWS, bool COLS, int G, bool SW = false, bool NORM = false, bool EXACT = false>
cudaError_t launch_tiles(const QParams& prm, cudaStream_t stream) {
  auto kern = quant_tile_kernel<FMT, ROWS, COLS, G, SW, NORM, EXACT>;
  constexpr uint32_t kQSmem = QCfg<SW>::kSmem;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // the attribute belongs to the context: set again in a new one
  static unsigned long long attr_ctx[64] = {};
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || attr_ctx[dev] != ctx) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
    if (e != cudaSuccess) return e;
    attr_ctx[dev] = ctx;
  }
  int sms = 0;
  e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  const int grid = prm.num_tiles < sms ? prm.num_tiles : sms;
  kern<<<grid, kQThreads, kQSmem, stream>>>(prm);
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_group(const QGroup& g, cudaStream_t stream) {
  auto kern = quant_group_kernel<FMT>;
  constexpr uint32_t kQSmem = QCfg<false>::kSmem;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static unsigned long long attr_ctx[64] = {};
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || attr_ctx[dev] != ctx) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
    if (e != cudaSuccess) return e;
    attr_ctx[dev] = ctx;
  }
  int sms = 0;
  e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  const int grid = g.num_tiles < sms ? g.num_tiles : sms;
  kern<<<grid, kQThreads, kQSmem, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_group(const QuantJob* jobs, int njobs, int fmt, cudaStream_t stream) {
  if (njobs < 1 || njobs > kQMaxJobs) return cudaErrorInvalidValue;
  QGroup g;
  std::memset(&g, 0, sizeof(g));
  int64_t total = 0;
  int n = 0;
  for (int i = 0; i < njobs; ++i) {
    const QuantJob& jb = jobs[i];
    if (jb.rows == 0 || jb.cols == 0) continue;
    QParams& p = g.job[n];
    if (!encode_x(&p.tmX, jb.x, jb.rows, jb.cols, jb.ldx)) return cudaErrorInvalidValue;
    p.M = jb.rows;
    p.K = jb.cols;
    p.q = static_cast<uint8_t*>(jb.q);
    p.s_rows = jb.s_rows;
    p.qt = static_cast<uint8_t*>(jb.qt);
    p.s_cols = jb.s_cols;
    p.lds_k = round_up128(jb.cols);
    p.tiles_k = static_cast<int>((jb.cols + 127) / 128);
    p.tk_magic = p.tiles_k > 0 ? 0xFFFFFFFFu / static_cast<uint32_t>(p.tiles_k) : 0u;
    if (jb.block) {
      p.lds_m = (jb.rows + 127) / 128;  // weight scales [K/128][ceil(N/128)]
      g.mode[n] = kQModeBlock;
    } else {
      p.lds_m = round_up128(jb.rows);
      g.mode[n] = (jb.q != nullptr ? kQModeRows : 0) | (jb.qt != nullptr ? kQModeCols : 0);
      if (g.mode[n] == 0) return cudaErrorInvalidValue;
    }
    total += ((jb.rows + 127) / 128) * static_cast<int64_t>(p.tiles_k);
    if (total > INT32_MAX) return cudaErrorInvalidValue;
    g.tile_end[n] = static_cast<int>(total);
    ++n;
  }
  if (n == 0) return cudaSuccess;
  g.njobs = n;
  g.num_tiles = static_cast<int>(total);
  cudaError_t e = device_status_word(&g.status);
  if (e != cudaSuccess) return e;
  g.limit_ns = 2000000000ull;
  return fmt == kFmtFp32 ? launch_group<kFmtFp32>(g, stream) : launch_group<kFmtUe8m0>(g, stream);
}

// X [M, K] -> any of: row-group codes q [M, K] + scales [K/G][round_up(M,128)]
// (q != nullptr), token-group codes qt [K, M] + scales [M/G][round_up(K,128)]
// (qt != nullptr; M % 128 == 0), for groups of G = 128 or (UE8M0 only) 32.
// K % 128 == 0 when q is requested.
cudaError_t launch_quant_tiles(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* s_rows,
                               void* qt, void* s_cols, int fmt, int group, cudaStream_t stream) {
  QParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!encode_x(&prm.tmX, x, M, K, ldx)) return cudaErrorInvalidValue;
  prm.M = M;
  prm.K = K;
  prm.q = static_cast<uint8_t*>(q);
  prm.s_rows = s_rows;
  prm.lds_m = round_up128(M);
  prm.qt = static_cast<uint8_t*>(qt);
  prm.s_cols = s_cols;
  prm.lds_k = round_up128(K);
  prm.tiles_k = static_cast<int>((K + 127) / 128);
  prm.tk_magic = prm.tiles_k > 0 ? 0xFFFFFFFFu / static_cast<uint32_t>(prm.tiles_k) : 0u;
  const int64_t tiles = ((M + 127) / 128) * prm.tiles_k;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  prm.num_tiles = static_cast<int>(tiles);
  int* status = nullptr;
  cudaError_t e = device_status_word(&status);
  if (e != cudaSuccess) return e;
  prm.status = status;
  prm.limit_ns = 2000000000ull;
  const bool rows = q != nullptr, cols = qt != nullptr;
  if (group == 32) {
    if (fmt != kFmtUe8m0) return cudaErrorInvalidValue;
    if (rows && cols) return launch_tiles<kFmtUe8m0, true, true, 32>(prm, stream);
    if (rows) return launch_tiles<kFmtUe8m0, true, false, 32>(prm, stream);
    return launch_tiles<kFmtUe8m0, false, true, 32>(prm, stream);
  }
  if (group != 128) return cudaErrorInvalidValue;
  if (fmt == kFmtFp32) {
    if (rows && cols) return launch_tiles<kFmtFp32, true, true, 128>(prm, stream);
    if (rows) return launch_tiles<kFmtFp32, true, false, 128>(prm, stream);
    return launch_tiles<kFmtFp32, false, true, 128>(prm, stream);
  }
  if (rows && cols) return launch_tiles<kFmtUe8m0, true, true, 128>(prm, stream);
  if (rows) return launch_tiles<kFmtUe8m0, true, false, 128>(prm, stream);
  return launch_tiles<kFmtUe8m0, false, true, 128>(prm, stream);
}

// SwiGLU fused with the quantization of its output: gu BF16 [M, 2F] holding
// [gate | up] -> h = silu(gate) * up (BF16, optionally stored to h [M, F]),
// quantized as quantize_act (q, s_rows) and, when qt != nullptr, as
// quantize_act_t (qt, s_cols).  F % 128 == 0; M % 128 == 0 when qt is set.
// exact: h rounded once from the exact value (swiglu_bf16x2<true>).
cudaError_t launch_swiglu_quant(const void* gu, int64_t M, int64_t F, int64_t ldgu, void* h, void* q, void* s_rows,
                                void* qt, void* s_cols, int fmt, bool exact, cudaStream_t stream) {
  QParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!encode_x(&prm.tmX, gu, M, 2 * F, ldgu)) return cudaErrorInvalidValue;
  prm.M = M;
  prm.K = F;
  prm.q = static_cast<uint8_t*>(q);
  prm.s_rows = s_rows;
  prm.lds_m = round_up128(M);
  prm.qt = static_cast<uint8_t*>(qt);
  prm.s_cols = s_cols;
  prm.lds_k = round_up128(F);
  prm.tiles_k = static_cast<int>(F / 128);
  prm.tk_magic = prm.tiles_k > 0 ? 0xFFFFFFFFu / static_cast<uint32_t>(prm.tiles_k) : 0u;
  const int64_t tiles = ((M + 127) / 128) * prm.tiles_k;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  prm.num_tiles = static_cast<int>(tiles);
  prm.up_off = F;
  prm.h = static_cast<uint16_t*>(h);
  prm.ldh = F;
  int* status = nullptr;
  cudaError_t e = device_status_word(&status);
  if (e != cudaSuccess) return e;
  prm.status = status;
  prm.limit_ns = 2000000000ull;
  const bool cols = qt != nullptr;
  if (exact) {
    if (fmt == kFmtFp32)
      return cols ? launch_tiles<kFmtFp32, true, true, 128, true, false, true>(prm, stream)
                  : launch_tiles<kFmtFp32, true, false, 128, true, false, true>(prm, stream);
    return cols ? launch_tiles<kFmtUe8m0, true, true, 128, true, false, true>(prm, stream)
                : launch_tiles<kFmtUe8m0, true, false, 128, true, false, true>(prm, stream);
  }
  if (fmt == kFmtFp32)
    return cols ? launch_tiles<kFmtFp32, true, true, 128, true>(prm, stream)
                : launch_tiles<kFmtFp32, true, false, 128, true>(prm, stream);
  return cols ? launch_tiles<kFmtUe8m0, true, true, 128, true>(prm, stream)
              : launch_tiles<kFmtUe8m0, true, false, 128, true>(prm, stream);
}

namespace {

// rstd[r] = 1 / sqrt(mean_k x[r, k]^2 + eps) in fp32 (IEEE square root and
// division): one warp per row, 8 values a lane per step, tree reduction.
__global__ void __launch_bounds__(256) rstd_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                                   float eps, float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= M) return;
  const uint16_t* row = x + r * ldx;
  float acc = 0.0f;
#pragma unroll 4
  for (int64_t k = 8 * lane; k < K; k += 256) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(row + k));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_lo(w[i]), b = bf16_hi(w[i]);
      acc = fmaf(a, a, acc);
      acc = fmaf(b, b, acc);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) rstd[r] = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(acc, static_cast<float>(K)) + eps));
}

// The same statistic in float64 (each x^2 exact, the sum, the mean, eps, the
// square root and the reciprocal in IEEE double): the exact RMSNorm's rstd.
__global__ void __launch_bounds__(256) rstd64_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                                                     int64_t ldx, double eps, double* __restrict__ rstd64) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= M) return;
  const uint16_t* row = x + r * ldx;
  double acc = 0.0;
#pragma unroll 4
  for (int64_t k = 8 * lane; k < K; k += 256) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(row + k));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double a = bf16_lo(w[i]), b = bf16_hi(w[i]);
      acc = fma(a, a, acc);
      acc = fma(b, b, acc);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) rstd64[r] = 1.0 / sqrt(acc / static_cast<double>(K) + eps);
}

// The RMSNorm tile pass, after the row statistics: rstd (fp32) for the
// default rounding, or rstd64 (float64, rstd == nullptr) for the exact one.
cudaError_t launch_norm_tiles(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, const float* rstd,
                              const double* rstd64, void* h, void* q, void* s_rows, void* qt, void* s_cols, int fmt,
                              cudaStream_t stream) {
  QParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!encode_x(&prm.tmX, x, M, K, ldx)) return cudaErrorInvalidValue;
  prm.M = M;
  prm.K = K;
  prm.q = static_cast<uint8_t*>(q);
  prm.s_rows = s_rows;
  prm.lds_m = round_up128(M);
  prm.qt = static_cast<uint8_t*>(qt);
  prm.s_cols = s_cols;
  prm.lds_k = round_up128(K);
  prm.tiles_k = static_cast<int>(K / 128);
  prm.tk_magic = prm.tiles_k > 0 ? 0xFFFFFFFFu / static_cast<uint32_t>(prm.tiles_k) : 0u;
  const int64_t tiles = ((M + 127) / 128) * prm.tiles_k;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  prm.num_tiles = static_cast<int>(tiles);
  prm.h = static_cast<uint16_t*>(h);
  prm.ldh = K;
  prm.rstd = rstd;
  prm.rstd64 = rstd64;
  prm.gamma = static_cast<const uint16_t*>(gamma);
  int* status = nullptr;
  const cudaError_t e = device_status_word(&status);
  if (e != cudaSuccess) return e;
  prm.status = status;
  prm.limit_ns = 2000000000ull;
  const bool cols = qt != nullptr;
  if (rstd64 != nullptr) {
    if (fmt == kFmtFp32)
      return cols ? launch_tiles<kFmtFp32, true, true, 128, false, true, true>(prm, stream)
                  : launch_tiles<kFmtFp32, true, false, 128, false, true, true>(prm, stream);
    return cols ? launch_tiles<kFmtUe8m0, true, true, 128, false, true, true>(prm, stream)
                : launch_tiles<kFmtUe8m0, true, false, 128, false, true, true>(prm, stream);
  }
  if (fmt == kFmtFp32)
    return cols ? launch_tiles<kFmtFp32, true, true, 128, false, true>(prm, stream)
                : launch_tiles<kFmtFp32, true, false, 128, false, true>(prm, stream);
  return cols ? launch_tiles<kFmtUe8m0, true, true, 128, false, true>(prm, stream)
              : launch_tiles<kFmtUe8m0, true, false, 128, false, true>(prm, stream);
}

}  // namespace

// RMSNorm fused with the quantization of its output: x BF16 [M, K] ->
// rstd [M] (fp32) -> h = x * rstd * gamma (BF16, optionally stored to h
// [M, K]), quantized as quantize_act (q, s_rows) and, when qt != nullptr, as
// quantize_act_t (qt, s_cols).  K % 128 == 0; M % 128 == 0 when qt is set.
cudaError_t launch_rmsnorm_quant(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
                                 float* rstd, void* h, void* q, void* s_rows, void* qt, void* s_cols, int fmt,
                                 cudaStream_t stream) {
  const int64_t blocks = (M + 7) / 8;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  rstd_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<const uint16_t*>(x), M, K, ldx, eps,
                                                                 rstd);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_norm_tiles(x, M, K, ldx, gamma, rstd, nullptr, h, q, s_rows, qt, s_cols, fmt, stream);
}

// The same with h rounded once from its exact value: rstd in float64
// (rstd64 [M], written), the fp32 products where their error bound decides
// the bf16 rounding, float64 for the rest (rmsnorm_exact_bf16x2).
cudaError_t launch_rmsnorm_quant_exact(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                       double eps, double* rstd64, void* h, void* q, void* s_rows, void* qt,
                                       void* s_cols, int fmt, cudaStream_t stream) {
  const int64_t blocks = (M + 7) / 8;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  rstd64_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<const uint16_t*>(x), M, K, ldx,
                                                                   eps, rstd64);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_norm_tiles(x, M, K, ldx, gamma, nullptr, rstd64, h, q, s_rows, qt, s_cols, fmt, stream);
}

}  // namespace fp8bq
