// quant_kernels.cu -- the three HBM-bound quantizers of the blockwise-FP8
// linear layer ("Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within
// $5090", section "方法": activations grouped by 128, weights in 128x128
// blocks).  Each reads BF16 once and writes E4M3 codes plus one scale per group
// or block; per element the work is a 2-byte read, a 1-byte write and a few
// ALU operations, so the kernels are sized for memory-level parallelism:
// 16-byte vector loads, several loads in flight per thread, coalesced stores.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "quant_math.cuh"

namespace fp8bq {

// ---------------------------------------------------------------------------
// 1x128 groups along the rows of X [M, K].
// A CTA owns 64 rows x one 128-column group; each half-warp owns one (row,
// group): 16 lanes x 8 bf16.  The amax is a 16-lane shuffle reduction.  Rows
// in [M, round_up(M,128)) only receive the neutral pad scale.
// ---------------------------------------------------------------------------
constexpr int kActRowsPerCta = 64;
constexpr int kActIters = 4;  // rows per half-warp

template <int FMT>
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                        int64_t K, int64_t ldx,
                                                        uint8_t* __restrict__ q,
                                                        void* __restrict__ scales, int64_t lds) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int64_t g = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kActRowsPerCta + warp * (2 * kActIters);
  const int64_t col = g * 128 + l16 * 8;

  uint4 v[kActIters];
#pragma unroll
  for (int i = 0; i < kActIters; ++i) {
    const int64_t r = row0 + 2 * i + half;
    if (r < M)
      v[i] = __ldcs(reinterpret_cast<const uint4*>(x + r * ldx + col));
    else
      v[i] = make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kActIters; ++i) {
    const int64_t r = row0 + 2 * i + half;
    float m = amax8(0.0f, v[i]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const GroupScale gs = make_scale<FMT>(m);
    if (r < M) {
      const uint2 c = quant8<FMT>(v[i], gs);
      *reinterpret_cast<uint2*>(q + r * K + col) = c;
      if (l16 == 0) store_scale<FMT>(scales, g * lds + r, gs);
    } else if (r < lds && l16 == 0) {
      store_neutral_scale<FMT>(scales, g * lds + r);
    }
  }
}

// ---------------------------------------------------------------------------
// 1x128 groups along the tokens: X [M, K] -> X^T codes [K, M].
// A CTA owns one 128-token group g and 64 columns c.  The BF16 tile passes
// through shared memory, 128 rows x 32 words (two bf16 per word); word p of
// row r lives at position p ^ (4 * (r / 16)), which keeps both the row-wise
// 16-byte stores and the column-wise 4-byte reads free of bank conflicts.
// In the column phase thread t owns columns 2p, 2p+1 (p = t / 8) and tokens
// 16j .. 16j+15 (j = t % 8): 8 lanes cover a group, amax over 3 shuffles, and
// each lane writes 16 consecutive codes of each of its two output rows.
// ---------------------------------------------------------------------------
constexpr int kTCols = 64;

template <int FMT>
__global__ void __launch_bounds__(256) quant_act_t_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                          int64_t K, int64_t ldx,
                                                          uint8_t* __restrict__ qt,
                                                          void* __restrict__ scales, int64_t lds) {
  __shared__ __align__(16) uint32_t tile[128][32];
  const int t = threadIdx.x;
  const int64_t g = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTCols;
  const int64_t m0 = g * 128;

  // load phase: 128 rows x 8 chunks of 16 B; thread t loads chunk t % 8 of
  // rows t / 8 + 32 i.
  {
    const int k = t & 7;
    const int64_t c = c0 + k * 8;
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (t >> 3) + 32 * i;
      if (c < K)
        v[i] = __ldcs(reinterpret_cast<const uint4*>(x + (m0 + r) * ldx + c));
      else
        v[i] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (t >> 3) + 32 * i;
      const int kk = k ^ (r >> 4);
      *reinterpret_cast<uint4*>(&tile[r][4 * kk]) = v[i];
    }
  }
  __syncthreads();

  const int p = t >> 3;  // column pair
  const int j = t & 7;   // token chunk
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = 16 * j + i;
    w[i] = tile[r][p ^ (4 * j)];
  }
  float m0v = 0.0f, m1v = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    m0v = fmaxf(m0v, fabsf(bf16_lo(w[i])));
    m1v = fmaxf(m1v, fabsf(bf16_hi(w[i])));
  }
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    m0v = fmaxf(m0v, __shfl_xor_sync(0xffffffffu, m0v, o));
    m1v = fmaxf(m1v, __shfl_xor_sync(0xffffffffu, m1v, o));
  }
  const GroupScale s0 = make_scale<FMT>(m0v);
  const GroupScale s1 = make_scale<FMT>(m1v);
  float xa[16], xb[16], ya[16], yb[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    xa[i] = bf16_lo(w[i]);
    xb[i] = bf16_hi(w[i]);
  }
  scaled_n<FMT, 16>(xa, s0, ya);
  scaled_n<FMT, 16>(xb, s1, yb);
  uint32_t a[4], b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i] = cvt_e4m3x2(ya[4 * i + 0], ya[4 * i + 1]) | (cvt_e4m3x2(ya[4 * i + 2], ya[4 * i + 3]) << 16);
    b[i] = cvt_e4m3x2(yb[4 * i + 0], yb[4 * i + 1]) | (cvt_e4m3x2(yb[4 * i + 2], yb[4 * i + 3]) << 16);
  }
  const int64_t ca = c0 + 2 * p;
  if (ca < K) {
    *reinterpret_cast<uint4*>(qt + ca * M + m0 + 16 * j) = make_uint4(a[0], a[1], a[2], a[3]);
    if (j == 0) store_scale<FMT>(scales, g * lds + ca, s0);
  } else if (ca < lds && j == 0) {
    store_neutral_scale<FMT>(scales, g * lds + ca);
  }
  if (ca + 1 < K) {
    *reinterpret_cast<uint4*>(qt + (ca + 1) * M + m0 + 16 * j) = make_uint4(b[0], b[1], b[2], b[3]);
    if (j == 0) store_scale<FMT>(scales, g * lds + ca + 1, s1);
  } else if (ca + 1 < lds && j == 0) {
    store_neutral_scale<FMT>(scales, g * lds + ca + 1);
  }
}

// ---------------------------------------------------------------------------
// 128x128 blocks of W [N, K].  One CTA per block: thread t loads chunk t % 16
// (8 bf16) of rows t / 16 + 16 i (i < 8), so a block's 32 KB is in registers
// while the CTA-wide amax is reduced (warp shuffles, then 8 partials through
// shared memory); the codes are then written straight from registers.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ w, int64_t N,
                                                           int64_t K, int64_t ldw,
                                                           uint8_t* __restrict__ q,
                                                           void* __restrict__ scales, int64_t nnb) {
  __shared__ float part[8];
  const int t = threadIdx.x;
  const int64_t nb = blockIdx.x;
  const int64_t kb = blockIdx.y;
  const int64_t col = kb * 128 + (t & 15) * 8;
  uint4 v[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = nb * 128 + (t >> 4) + 16 * i;
    if (r < N)
      v[i] = __ldcs(reinterpret_cast<const uint4*>(w + r * ldw + col));
    else
      v[i] = make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) m = amax8(m, v[i]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((t & 31) == 0) part[t >> 5] = m;
  __syncthreads();
  m = part[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, part[i]);
  const GroupScale gs = make_scale<FMT>(m);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = nb * 128 + (t >> 4) + 16 * i;
    if (r < N) *reinterpret_cast<uint2*>(q + r * K + col) = quant8<FMT>(v[i], gs);
  }
  if (t == 0) store_scale<FMT>(scales, kb * nnb + nb, gs);
}

// --------------------------------------------------------------- launchers --
cudaError_t launch_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                             int fmt, cudaStream_t stream) {
  const int64_t lds = round_up128(M);
  const dim3 grid(static_cast<unsigned>(lds / kActRowsPerCta), static_cast<unsigned>(K / 128));
  const auto* xp = static_cast<const uint16_t*>(x);
  auto* qp = static_cast<uint8_t*>(q);
  if (fmt == kFmtFp32)
    quant_act_kernel<kFmtFp32><<<grid, 256, 0, stream>>>(xp, M, K, ldx, qp, scales, lds);
  else
    quant_act_kernel<kFmtUe8m0><<<grid, 256, 0, stream>>>(xp, M, K, ldx, qp, scales, lds);
  return cudaGetLastError();
}

cudaError_t launch_quant_act_t(const void* x, int64_t M, int64_t K, int64_t ldx, void* qt,
                               void* scales, int fmt, cudaStream_t stream) {
  const int64_t lds = round_up128(K);
  const dim3 grid(static_cast<unsigned>(lds / kTCols), static_cast<unsigned>(M / 128));
  const auto* xp = static_cast<const uint16_t*>(x);
  auto* qp = static_cast<uint8_t*>(qt);
  if (fmt == kFmtFp32)
    quant_act_t_kernel<kFmtFp32><<<grid, 256, 0, stream>>>(xp, M, K, ldx, qp, scales, lds);
  else
    quant_act_t_kernel<kFmtUe8m0><<<grid, 256, 0, stream>>>(xp, M, K, ldx, qp, scales, lds);
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const void* w, int64_t N, int64_t K, int64_t ldw, void* q,
                                void* scales, int fmt, cudaStream_t stream) {
  const int64_t nnb = (N + 127) / 128;
  const dim3 grid(static_cast<unsigned>(nnb), static_cast<unsigned>(K / 128));
  const auto* wp = static_cast<const uint16_t*>(w);
  auto* qp = static_cast<uint8_t*>(q);
  if (fmt == kFmtFp32)
    quant_weight_kernel<kFmtFp32><<<grid, 256, 0, stream>>>(wp, N, K, ldw, qp, scales, nnb);
  else
    quant_weight_kernel<kFmtUe8m0><<<grid, 256, 0, stream>>>(wp, N, K, ldw, qp, scales, nnb);
  return cudaGetLastError();
}

}  // namespace fp8bq
