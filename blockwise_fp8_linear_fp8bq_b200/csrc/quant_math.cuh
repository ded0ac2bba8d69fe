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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// amax update over the two bf16 values packed in w.
__device__ __forceinline__ float amax2(float m, uint32_t w) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))));
}

// Two fp32 -> two E4M3 bytes, round-to-nearest-even with saturation to +-448;
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Per-group quantization parameters.  FP32 scales: `s` and, when s is a
// normal number well above the underflow range, `mul` = RN(1/s) (else 0).
// UE8M0: `mul` = 2^-e exactly.
struct GroupScale {
  float s;        // FP32 scale value (FP32 format)
  float mul;      // RN(1/s) (FP32 format) or 2^-e (UE8M0 format)
  uint32_t byte;  // e + 127 (UE8M0 format)
};

template <int FMT>
__device__ __forceinline__ GroupScale make_scale(float amax) {
  GroupScale g;
  if constexpr (FMT == kFmtFp32) {
    g.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    g.mul = (g.s >= 0x1p-125f) ? __frcp_rn(g.s) : 0.0f;
    g.byte = 0;
  } else {
    // From the IEEE fields of amax = 1.f * 2^E:  448 = 1.75 * 2^8, so
    // amax <= 448 * 2^(E-8) exactly when the significand is <= 1.75
    // (fraction field <= 0x600000); otherwise one more power is needed.
    // Subnormal amax lies far below 448 * 2^-127 and takes the clamp.
    const uint32_t u = __float_as_uint(amax);
    const int ef = static_cast<int>((u >> 23) & 0xFF);
    int e;
    if (amax == 0.0f) {
      e = 0;
    } else if (ef == 0) {
      e = -127;
    } else {
      e = (ef - 127) - 8 + (((u & 0x7FFFFFu) > 0x600000u) ? 1 : 0);
      e = e < -127 ? -127 : (e > 127 ? 127 : e);
    }
    g.s = 0.0f;
    g.mul = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal for e in [-127,127)
    g.byte = static_cast<uint32_t>(e + 127);
  }
  return g;
}

// fl32(x / s) as far as the E4M3 encoder can tell.  q = RN(x * RN(1/s)) is
// within 2.5 fp32 ulps of the IEEE quotient RN(x / s) (two roundings of
// relative size 2^-24 each, plus the quotient's own half ulp).  Every decision
// boundary of the saturating round-to-nearest-even E4M3 encoder -- a midpoint
// between neighbouring E4M3 values, including 2^-10 between 0 and the least
// subnormal -- has at most 5 significant bits, so bits 18..0 of its fp32
// encoding are zero.  When q is more than 8 encodings away from every such
// value, q and RN(x / s) lie strictly on the same side of every boundary and
// encode to the same E4M3 code; otherwise (a fraction ~3e-5 of the values)
// the IEEE division is taken.  Groups whose scale is too small for a finite
// reciprocal (mul == 0) always take the IEEE division.
__device__ __forceinline__ bool near_e4m3_boundary(float q) {
  return ((__float_as_uint(q) + 8u) & 0x7FFFFu) <= 16u;
}

template <int FMT>
__device__ __forceinline__ float scaled(float x, const GroupScale& g) {
  if constexpr (FMT == kFmtFp32) {
    if (g.mul == 0.0f) return __fdiv_rn(x, g.s);
    const float q = x * g.mul;
    return near_e4m3_boundary(q) ? __fdiv_rn(x, g.s) : q;
  } else {
    return x * g.mul;
  }
}

// n values -> their scaled quotients; the IEEE division, when any value
// needs it, runs in one rarely taken branch rather than per element.
template <int FMT, int N>
__device__ __forceinline__ void scaled_n(const float (&x)[N], const GroupScale& g, float (&y)[N]) {
  if constexpr (FMT == kFmtFp32) {
    bool slow = (g.mul == 0.0f);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      y[i] = x[i] * g.mul;
      slow |= near_e4m3_boundary(y[i]);
    }
    if (__builtin_expect(slow, 0)) {
#pragma unroll
      for (int i = 0; i < N; ++i) y[i] = scaled<FMT>(x[i], g);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) y[i] = x[i] * g.mul;
  }
}

// Eight bf16 (one uint4) -> eight E4M3 codes (one uint2).
template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, const GroupScale& g) {
  float x[8], y[8];
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
  scaled_n<FMT, 8>(x, g, y);
  uint2 r;
  r.x = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
  r.y = cvt_e4m3x2(y[4], y[5]) | (cvt_e4m3x2(y[6], y[7]) << 16);
  return r;
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
