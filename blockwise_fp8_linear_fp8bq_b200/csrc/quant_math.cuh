// quant_math.cuh -- per-element arithmetic of the blockwise-FP8 quantizers,
// shared by the three quantizer kernels and the GEMM's fused quantize-on-load
// so that all of them produce bit-identical codes and scales.
//
// Method ("Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090",
// section "方法"): 1x128 activation groups and 128x128 weight blocks, one scale
// per group or block, E4M3 codes; "MXFP8 on Blackwell" read as power-of-two
// (UE8M0) scales.
//   FP32 scale : s = fl32(amax / 448) (1 for an all-zero group);
//                q = E4M3 round-to-nearest-even, saturating, of fl32(x / s).
//   UE8M0 scale: e = least integer with amax <= 448 * 2^e, in [-127, 127]
//                (0 for an all-zero group); q = E4M3_RNE_sat(x * 2^-e).
#pragma once
#include <cstdint>

namespace fp8bq {

constexpr int kFmtFp32 = 0;
constexpr int kFmtUe8m0 = 1;
constexpr int kFmtMx = 2;  // GEMM only: UE8M0 scales on 1x32 blocks (MX)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// amax update over the two bf16 values packed in w.
__device__ __forceinline__ float amax2(float m, uint32_t w) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))));
}

// Per bf16 half: max(|a|, |b|) in magnitude; the sign bits of the result are
// those of a XOR b and carry no meaning (mask them with 0x7FFF7FFF).  One
// instruction per two values for the group amax of finite inputs.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Two fp32 -> two E4M3 bytes, round-to-nearest-even with saturation to +-448;
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Per-group quantization parameters.  FP32 scales: `s` and r = RN(1/s) when
// s is well inside the normal range (else 0).  UE8M0: `mul` = 2^-e exactly.
struct GroupScale {
  float s;        // FP32 scale value (FP32 format)
  float r;        // FP32 format: RN(1/s), or 0 for s < 2^-125
  float mul;      // 2^-e (UE8M0 format); unused for FP32
  uint32_t byte;  // e + 127 (UE8M0 format)
};

template <int FMT>
__device__ __forceinline__ GroupScale make_scale(float amax) {
  GroupScale g;
  if constexpr (FMT == kFmtFp32) {
    g.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    g.r = (g.s >= 0x1p-125f) ? __frcp_rn(g.s) : 0.0f;
    g.mul = 0.0f;
    g.byte = 0;
  } else {
    // From the IEEE fields of amax = 1.f * 2^E (amax >= 0, finite):  448 =
    // 1.75 * 2^8, so amax <= 448 * 2^(E-8) exactly when the significand is
    // <= 1.75 (fraction field <= 0x600000); otherwise one more power is
    // needed.  Adding 0x1FFFFF to the bits carries into the exponent field
    // exactly when the fraction exceeds 0x600000, so the biased result
    // e + 127 = E + 127 - 8 + carry is one add and one shift.  Subnormal (or
    // tiny) amax lies below 448 * 2^-127: the clamp at 0 gives e = -127.
    // e never exceeds 120 for finite amax, so no upper clamp is needed.
    const uint32_t u = __float_as_uint(amax);
    int biased = static_cast<int>((u + 0x1FFFFFu) >> 23) - 8;
    biased = biased < 0 ? 0 : biased;
    if (amax == 0.0f) biased = 127;
    const int e = biased - 127;
    g.s = 0.0f;
    g.r = 0.0f;
    g.mul = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal for e in [-127,127)
    g.byte = static_cast<uint32_t>(e + 127);
  }
  return g;
}

// The code of fl32(x / s), found without a division.  With r = RN(1/s) and
// q = x / s, y0 = RN(x r) lies within 1.5 ulp of q.  One correction
// y1 = RN(y0 - r RN(s y0 - x)) is then within 1/2 ulp + 2^-22 ulp of q, i.e.
// a faithful rounding, for which the residual s y1 - x is exact (fused
// multiply-add); Markstein's theorem (P. Markstein, IBM J. Res. Dev. 34(1),
// 1990; M. Cornea, J. Harrison, P. Markstein, ARITH-14, 1999) then gives
// y2 = RN(y1 - r (s y1 - x)) = RN(q) when r = RN(1/s), barring overflow and
// underflow.  |q| <= 448 rules out overflow; results small enough to
// underflow all encode to a signed zero either way.  Residuals are taken as
// s y - x so that fma(s, +-0, -+0) = +0 and fma(-r, +0, +-0) = +-0 keep the
// sign of a zero input.  Groups with s < 2^-125 (r = 0) set `slow`; the
// caller then recomputes with the IEEE division (quant8_exact).
template <int FMT>
__device__ __forceinline__ uint32_t quant2_fast(float2 xx, const GroupScale& g) {
  if constexpr (FMT == kFmtFp32) {
    const float2 r2 = make_float2(g.r, g.r);
    const float2 nr2 = make_float2(-g.r, -g.r);
    const float2 s2 = make_float2(g.s, g.s);
    const float2 nx = make_float2(-xx.x, -xx.y);
    float2 y = __fmul2_rn(xx, r2);
    float2 e = __ffma2_rn(s2, y, nx);
    y = __ffma2_rn(nr2, e, y);
    e = __ffma2_rn(s2, y, nx);
    y = __ffma2_rn(nr2, e, y);
    return cvt_e4m3x2(y.x, y.y);
  } else {
    // x * 2^-e is exact (barring underflow to values that encode to zero)
    const float2 y = __fmul2_rn(xx, make_float2(g.mul, g.mul));
    return cvt_e4m3x2(y.x, y.y);
  }
}

// Two values -> two E4M3 codes (low byte: xx.x); see quant2_fast.  A group
// whose scale is too small for the division-free quotient sets `slow`.
template <int FMT>
__device__ __forceinline__ uint32_t quant2_fast(float2 xx, const GroupScale& g, bool& slow) {
  if constexpr (FMT == kFmtFp32) slow |= (g.r == 0.0f);
  return quant2_fast<FMT>(xx, g);
}

template <int FMT>
__device__ __forceinline__ uint2 quant8_fast(const uint4& v, const GroupScale& g, bool& slow) {
  uint32_t c[4];
  c[0] = quant2_fast<FMT>(make_float2(bf16_lo(v.x), bf16_hi(v.x)), g);
  c[1] = quant2_fast<FMT>(make_float2(bf16_lo(v.y), bf16_hi(v.y)), g);
  c[2] = quant2_fast<FMT>(make_float2(bf16_lo(v.z), bf16_hi(v.z)), g);
  c[3] = quant2_fast<FMT>(make_float2(bf16_lo(v.w), bf16_hi(v.w)), g);
  if constexpr (FMT == kFmtFp32) slow |= (g.r == 0.0f);
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Eight bf16 -> eight E4M3 codes of fl32(x / s) with the IEEE division.  Kept
// out of line: it runs only for groups of tiny scale, and inlined copies would
// raise every kernel's register count.
template <int FMT>
static __device__ __noinline__ uint2 quant8_exact_outlined(uint4 v, float s, float mul) {
  float y[8];
  const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = (FMT == kFmtFp32) ? __fdiv_rn(x[i], s) : x[i] * mul;
  uint2 r;
  r.x = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
  r.y = cvt_e4m3x2(y[4], y[5]) | (cvt_e4m3x2(y[6], y[7]) << 16);
  return r;
}

template <int FMT>
__device__ __forceinline__ uint2 quant8_exact(const uint4& v, const GroupScale& g) {
  return quant8_exact_outlined<FMT>(v, g.s, g.mul);
}

// Eight bf16 -> eight E4M3 codes (single-value callers; fused quantize-on-load).
template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, const GroupScale& g) {
  return quant8_exact<FMT>(v, g);
}

// Group scale for the group whose amax sits in lane `src` of `amax`, computed
// once per warp: every lane computes the scale of one group (its own amax) and
// lanes fetch the result from `src`.
template <int FMT>
__device__ __forceinline__ GroupScale fetch_scale(const GroupScale& mine, int src) {
  GroupScale g;
  if constexpr (FMT == kFmtFp32) {
    g.s = __shfl_sync(0xffffffffu, mine.s, src);
    g.r = __shfl_sync(0xffffffffu, mine.r, src);
    g.mul = 0.0f;
    g.byte = 0;
  } else {
    g.s = 0.0f;
    g.r = 0.0f;
    g.mul = __shfl_sync(0xffffffffu, mine.mul, src);
    g.byte = __shfl_sync(0xffffffffu, mine.byte, src);
  }
  return g;
}

__device__ __forceinline__ float amax8(float m, const uint4& v) {
  return amax2(amax2(amax2(amax2(m, v.x), v.y), v.z), v.w);
}

template <int FMT>
__device__ __forceinline__ void store_scale(void* scales, int64_t idx, const GroupScale& g) {
  if constexpr (FMT == kFmtFp32)
    static_cast<float*>(scales)[idx] = g.s;
  else
    static_cast<uint8_t*>(scales)[idx] = static_cast<uint8_t>(g.byte);
}

template <int FMT>
__device__ __forceinline__ void store_neutral_scale(void* scales, int64_t idx) {
  if constexpr (FMT == kFmtFp32)
    static_cast<float*>(scales)[idx] = 1.0f;
  else
    static_cast<uint8_t*>(scales)[idx] = 127;
}

}  // namespace fp8bq
