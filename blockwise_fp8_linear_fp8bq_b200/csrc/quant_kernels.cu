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
__global__ void __launch_bounds__(256, FMT == kFmtFp32 ? 4 : 5) quant_act_kernel(const uint16_t* __restrict__ x, int64_t M,
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
  // amax of each (iteration, half) group; lane 2 i + h then computes the
  // scale of group (i, h) and every lane fetches the scales it needs.
  float m[kActIters];
#pragma unroll
  for (int i = 0; i < kActIters; ++i) {
    m[i] = amax8(0.0f, v[i]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
  }
  GroupScale gs[kActIters];
  if constexpr (FMT == kFmtFp32) {
    // an IEEE division and reciprocal per group: computed once per warp
    float mine = 0.0f;
#pragma unroll
    for (int i = 0; i < kActIters; ++i) {
      const float mi = __shfl_sync(0xffffffffu, m[i], (lane & 1) * 16);
      if ((lane >> 1) == i) mine = mi;
    }
    const GroupScale gmine = make_scale<FMT>(mine);
#pragma unroll
    for (int i = 0; i < kActIters; ++i) gs[i] = fetch_scale<FMT>(gmine, 2 * i + half);
  } else {
#pragma unroll
    for (int i = 0; i < kActIters; ++i) gs[i] = make_scale<FMT>(m[i]);
  }

  uint2 c[kActIters];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < kActIters; ++i) c[i] = quant8_fast<FMT>(v[i], gs[i], slow);
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int i = 0; i < kActIters; ++i) c[i] = quant8_exact<FMT>(v[i], gs[i]);
  }
#pragma unroll
  for (int i = 0; i < kActIters; ++i) {
    const int64_t r = row0 + 2 * i + half;
    if (r < M) {
      *reinterpret_cast<uint2*>(q + r * K + col) = c[i];
      if (l16 == 0) store_scale<FMT>(scales, g * lds + r, gs[i]);
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
__global__ void __launch_bounds__(256, FMT == kFmtFp32 ? 4 : 5) quant_act_t_kernel(const uint16_t* __restrict__ x, int64_t M,
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
  // The warp holds 8 groups (4 column pairs x 2 columns); lane 2 a + b
  // computes the scale of column b of pair a, the others fetch it.
  GroupScale s0, s1;
  if constexpr (FMT == kFmtFp32) {
    const int lane = t & 31;
    const int a4 = lane >> 3;  // pair within the warp
    float mine = 0.0f;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float t0 = __shfl_sync(0xffffffffu, m0v, 8 * a);
      const float t1 = __shfl_sync(0xffffffffu, m1v, 8 * a);
      if (lane == 2 * a) mine = t0;
      if (lane == 2 * a + 1) mine = t1;
    }
    const GroupScale gmine = make_scale<FMT>(mine);
    s0 = fetch_scale<FMT>(gmine, 2 * a4);
    s1 = fetch_scale<FMT>(gmine, 2 * a4 + 1);
  } else {
    s0 = make_scale<FMT>(m0v);
    s1 = make_scale<FMT>(m1v);
  }
  uint4 wa[2], wb[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    // columns 2p (low halves) and 2p+1 (high halves) of tokens 8h .. 8h+7
    wa[h] = make_uint4((w[8 * h + 0] & 0xFFFFu) | (w[8 * h + 1] << 16), (w[8 * h + 2] & 0xFFFFu) | (w[8 * h + 3] << 16),
                       (w[8 * h + 4] & 0xFFFFu) | (w[8 * h + 5] << 16), (w[8 * h + 6] & 0xFFFFu) | (w[8 * h + 7] << 16));
    wb[h] = make_uint4((w[8 * h + 0] >> 16) | (w[8 * h + 1] & 0xFFFF0000u), (w[8 * h + 2] >> 16) | (w[8 * h + 3] & 0xFFFF0000u),
                       (w[8 * h + 4] >> 16) | (w[8 * h + 5] & 0xFFFF0000u), (w[8 * h + 6] >> 16) | (w[8 * h + 7] & 0xFFFF0000u));
  }
  uint2 ca2[2], cb2[2];
  bool slow = false;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    ca2[h] = quant8_fast<FMT>(wa[h], s0, slow);
    cb2[h] = quant8_fast<FMT>(wb[h], s1, slow);
  }
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ca2[h] = quant8_exact<FMT>(wa[h], s0);
      cb2[h] = quant8_exact<FMT>(wb[h], s1);
    }
  }
  uint32_t a[4] = {ca2[0].x, ca2[0].y, ca2[1].x, ca2[1].y};
  uint32_t b[4] = {cb2[0].x, cb2[0].y, cb2[1].x, cb2[1].y};
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
  uint2 c[8];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = quant8_fast<FMT>(v[i], gs, slow);
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = quant8_exact<FMT>(v[i], gs);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = nb * 128 + (t >> 4) + 16 * i;
    if (r < N) *reinterpret_cast<uint2*>(q + r * K + col) = c[i];
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
