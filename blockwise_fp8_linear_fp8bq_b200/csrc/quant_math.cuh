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

// Per-group quantization parameters.  FP32 scales: `s`, and the bracketing
// multipliers mlo / mhi = RN(1/s) * (1 -/+ 2^-20) when s is well above the
// underflow range (else 0).  UE8M0: `mul` = 2^-e exactly.
struct GroupScale {
  float s;        // FP32 scale value (FP32 format)
  float mul;      // 2^-e (UE8M0 format); unused for FP32
  float mlo, mhi; // FP32 format: bracketing multipliers
  uint32_t byte;  // e + 127 (UE8M0 format)
};

template <int FMT>
__device__ __forceinline__ GroupScale make_scale(float amax) {
  GroupScale g;
  if constexpr (FMT == kFmtFp32) {
    g.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    const float r = (g.s >= 0x1p-125f) ? __frcp_rn(g.s) : 0.0f;
    g.mul = 0.0f;
    g.mlo = r * (1.0f - 0x1p-20f);
    g.mhi = r * (1.0f + 0x1p-20f);
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
    g.mlo = g.mhi = 0.0f;
    g.byte = static_cast<uint32_t>(e + 127);
  }
  return g;
}

// The code of fl32(x / s), found without a division.  With r = RN(1/s)
// (relative error <= 2^-24), q_lo = RN(x * RN(r (1 - 2^-20))) and
// q_hi = RN(x * RN(r (1 + 2^-20))) lie within (1 -/+ 2^-20)(1 +/- 3 * 2^-24)
// of x / s, so |q_lo| < |RN(x / s)| < |q_hi| with the same sign.  The E4M3
// encoder (round to nearest even, saturating) is monotonic, so when q_lo and
// q_hi encode to the same code, so does RN(x / s).  Otherwise -- a decision
// boundary lies in the bracket, for about one value in 2^16 -- the caller
// recomputes with the IEEE division (quant8_exact), as it does for groups
// whose scale has no finite reciprocal (mlo == 0).
template <int FMT>
__device__ __forceinline__ uint2 quant8_fast(const uint4& v, const GroupScale& g, bool& slow) {
  float x[8];
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
  uint2 r;
  if constexpr (FMT == kFmtFp32) {
    uint2 h;
    r.x = cvt_e4m3x2(x[0] * g.mlo, x[1] * g.mlo) | (cvt_e4m3x2(x[2] * g.mlo, x[3] * g.mlo) << 16);
    r.y = cvt_e4m3x2(x[4] * g.mlo, x[5] * g.mlo) | (cvt_e4m3x2(x[6] * g.mlo, x[7] * g.mlo) << 16);
    h.x = cvt_e4m3x2(x[0] * g.mhi, x[1] * g.mhi) | (cvt_e4m3x2(x[2] * g.mhi, x[3] * g.mhi) << 16);
    h.y = cvt_e4m3x2(x[4] * g.mhi, x[5] * g.mhi) | (cvt_e4m3x2(x[6] * g.mhi, x[7] * g.mhi) << 16);
    slow |= (r.x != h.x) | (r.y != h.y) | (g.mlo == 0.0f);
  } else {
    r.x = cvt_e4m3x2(x[0] * g.mul, x[1] * g.mul) | (cvt_e4m3x2(x[2] * g.mul, x[3] * g.mul) << 16);
    r.y = cvt_e4m3x2(x[4] * g.mul, x[5] * g.mul) | (cvt_e4m3x2(x[6] * g.mul, x[7] * g.mul) << 16);
  }
  return r;
}

// Eight bf16 -> eight E4M3 codes of fl32(x / s) with the IEEE division for
// every value near a boundary.  Kept out of line: it runs only on the rare
// exact path, and inlined copies would raise every kernel's register count.
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
  g.s = __shfl_sync(0xffffffffu, mine.s, src);
  g.mul = __shfl_sync(0xffffffffu, mine.mul, src);
  g.mlo = __shfl_sync(0xffffffffu, mine.mlo, src);
  g.mhi = __shfl_sync(0xffffffffu, mine.mhi, src);
  g.byte = __shfl_sync(0xffffffffu, mine.byte, src);
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
