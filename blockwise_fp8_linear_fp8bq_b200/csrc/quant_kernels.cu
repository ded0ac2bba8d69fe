// quant_kernels.cu -- the 128x128 weight-block quantizer of the blockwise-FP8
// linear layer ("Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within
// $5090", section "方法": weights in 128x128 blocks).  It reads BF16 once and
// writes E4M3 codes plus one scale per block; the activation quantizers are in
// quant_tiles.cu.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "quant_math.cuh"

namespace fp8bq {

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
  // packed |max| (two bf16 values per instruction), reduced over the warp
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    m2 = absmax_bf16x2(absmax_bf16x2(m2, v[i].x), absmax_bf16x2(v[i].y, absmax_bf16x2(v[i].z, v[i].w)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  m2 &= 0x7FFF7FFFu;
  m = fmaxf(bf16_lo(m2), bf16_hi(m2));
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
