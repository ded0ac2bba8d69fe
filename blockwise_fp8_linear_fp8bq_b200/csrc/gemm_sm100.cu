// gemm_sm100.cu -- blockwise-FP8 GEMM on the 5th-generation tensor cores.
//
//   D[m, n] = sum_kb  sA(m, kb) * sB(n, kb) * sum_{k in kb} qA[m, k] * qB[n, k]
//
// with 128-long K blocks kb, E4M3 codes q, FP32 accumulation and one BF16
// rounding at the end: the linear layer of "Puro-2B: Poor Lab's Qwen2-1.5B
// Trained on RTX 5090 within $5090" (section "方法": 1x128 activation groups,
// 128x128 weight blocks, MXFP8 on Blackwell) and of the ModelScope post's
// section "精度：FP8 分块量化与净效率收益" (the linear layers' matmuls in FP8).
//
// Kernel shape (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: A and B K-block tiles (128-byte swizzle) and the
//               raw scale vectors of each K block, into a 4-stage ring.
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma.
//   warp 2      scale staging: writes the 128x128-block scale of B into the
//               ring (FP32 path) or rearranges the UE8M0 scales into the
//               layout tcgen05.cp copies into tensor memory (block-scaled path).
//   warps 3-10  epilogue; each owns 32 rows (its TMEM lane quarter) x 128
//               columns of the tile.
// FP32 scales ("promotion" path): each K block's MMAs write a fresh partial
// product into one of two 256-column TMEM buffers; the epilogue warps load it,
// multiply by sA * sB and add it into FP32 register accumulators while the
// tensor core fills the other buffer.  UE8M0 scales: the block-scaled MMA
// (kind::mxf8f6f4.block_scale) applies the power-of-two scales itself and
// accumulates the whole K extent in one TMEM buffer; the epilogue drains it
// into registers once per tile and frees it before converting and storing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace fp8bq {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int STAGES = 4;
constexpr int kThreads = 352;  // 11 warps
constexpr int kEpiWarp0 = 3;
constexpr int kEpiWarps = 8;
constexpr int kTmemCols = 512;
constexpr int kGroupM = 8;  // M blocks per raster group (L2 reuse of B)

constexpr uint32_t kTileABytes = BM * BK;  // 16 KB
constexpr uint32_t kTileBBytes = BN * BK;  // 32 KB
// per-stage scale slot
constexpr uint32_t kSlotRawA = 0;      // 128 FP32 scales (512 B) or 128 UE8M0 bytes
constexpr uint32_t kSlotRawB = 512;    // 256 FP32 scales (1 KB) or 256 UE8M0 bytes
constexpr uint32_t kSlotBlk = 1536;    // two 128x128-block scales of B (FP32 path)
constexpr uint32_t kSlotTm = 1664;     // 1536 B: tensor-memory images of the UE8M0 scales
constexpr uint32_t kSlotBytes = 3200;  // multiple of 128

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + STAGES * kTileABytes;
constexpr uint32_t kOffSlot = kOffB + STAGES * kTileBBytes;
constexpr uint32_t kOffBar = kOffSlot + STAGES * kSlotBytes;
// barriers: full[S], empty[S], sfready[S], scempty[S], tfull[2], tempty[2], final
constexpr uint32_t kNumBars = 4 * STAGES + 5;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-B alignment

// TMEM columns: FP32 path: partial buffers at 0 and 256.  UE8M0 path: the
// accumulator at 0..255, then per stage s the A scales at 256 + 16 s (4 cols)
// and the B scales at 256 + 16 s + 8 (8 cols).
constexpr uint32_t kTmemSf = 256;

constexpr int kTimeoutProducer = 1;
constexpr int kTimeoutMma = 2;
constexpr int kTimeoutScale = 3;
constexpr int kTimeoutEpilogue = 4;
constexpr int kTimeoutTeardown = 5;

struct Params {
  CUtensorMap tmA;
  CUtensorMap tmB;
  const void* sA;        // A row-group scales [K/128][lds_a]
  const void* sB;        // B scales (row groups or blocks)
  int64_t sa_stride_k;   // = lds_a
  int64_t sb_stride_k;
  int64_t sb_stride_r;
  int64_t sb_len;        // row groups: lds_b (row stride of B's scale array)
  int64_t nb_blocks;     // 128x128 blocks: number of B row blocks (ceil(N/128))
  uint16_t* D;
  int64_t ldd;
  int M, N, K;
  int num_m, num_n, num_tiles, num_kb;
  int* status;
  uint64_t limit_ns;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
  const int group = tile / (kGroupM * num_n);
  const int first_m = group * kGroupM;
  const int gsz = min(kGroupM, num_m - first_m);
  const int r = tile - group * kGroupM * num_n;
  mb = first_m + r % gsz;
  nb = r / gsz;
}

// Scales of B's two 128-row blocks for 32 consecutive K blocks: lane l holds
// K block base + l.  Used by the scale-staging warp for 128x128-block B.
__device__ __forceinline__ void load_block_scales(const Params& p, int nb, int kb0, bool fp32,
                                                  uint32_t& v0, uint32_t& v1) {
  const int lane = threadIdx.x & 31;
  const int kb = kb0 + lane;
  v0 = 0;
  v1 = 0;
  if (kb < p.num_kb) {
    const int64_t r0 = 2 * static_cast<int64_t>(nb);
    const int64_t i0 = kb * p.sb_stride_k + r0 * p.sb_stride_r;
    const int64_t i1 = i0 + p.sb_stride_r;
    if (fp32) {
      const uint32_t* s = static_cast<const uint32_t*>(p.sB);
      v0 = __ldg(s + i0);
      v1 = (r0 + 1 < p.nb_blocks) ? __ldg(s + i1) : 0x3F800000u;
    } else {
      const uint8_t* s = static_cast<const uint8_t*>(p.sB);
      v0 = __ldg(s + i0);
      v1 = (r0 + 1 < p.nb_blocks) ? __ldg(s + i1) : 127u;
    }
  }
}

template <int FMT, bool B_KMAJOR, bool B_ROW>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool kFp32 = (FMT == kFmtFp32);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto full_bar = [&](int s) { return bar(s); };
  auto empty_bar = [&](int s) { return bar(STAGES + s); };
  auto sfready_bar = [&](int s) { return bar(2 * STAGES + s); };
  auto scempty_bar = [&](int s) { return bar(3 * STAGES + s); };
  auto tfull_bar = [&](int b) { return bar(4 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar(4 * STAGES + 2 + b); };
  const uint32_t final_bar = bar(4 * STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  const WaitGuard guard{abort_flag, p.status, p.limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sfready_bar(s), 1);
      mbar_init(scempty_bar(s), kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int KB = p.num_kb;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tmA);
      prefetch_tensormap(&p.tmB);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.num_m, p.num_n, mb, nb);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, guard, kTimeoutProducer)) { ok = false; break; }
          if (kFp32 && !mbar_wait(scempty_bar(s), ph ^ 1, guard, kTimeoutProducer)) { ok = false; break; }
          uint8_t* slot = smem + kOffSlot + s * kSlotBytes;
          uint32_t tx = kTileABytes + kTileBBytes;
          const uint32_t a_sc_bytes = kFp32 ? 512u : 128u;
          uint32_t b_sc_bytes = 0;
          if (B_ROW) {
            const int64_t left = p.sb_len - static_cast<int64_t>(nb) * BN;
            const int64_t n = left < BN ? left : BN;  // a multiple of 128
            b_sc_bytes = static_cast<uint32_t>(n) * (kFp32 ? 4u : 1u);
          }
          tx += a_sc_bytes + b_sc_bytes;
          mbar_arrive_expect_tx(full_bar(s), tx);
          const uint32_t sa = smem_u32(smem + kOffA + s * kTileABytes);
          const uint32_t sb = smem_u32(smem + kOffB + s * kTileBBytes);
          tma_load_2d(sa, &p.tmA, full_bar(s), kb * BK, mb * BM);
          if (B_KMAJOR) {
            tma_load_2d(sb, &p.tmB, full_bar(s), kb * BK, nb * BN);
          } else {
            tma_load_2d(sb, &p.tmB, full_bar(s), nb * BN, kb * BK);
            tma_load_2d(sb + kTileBBytes / 2, &p.tmB, full_bar(s), nb * BN + 128, kb * BK);
          }
          const uint8_t* ga = static_cast<const uint8_t*>(p.sA) +
                              (kb * p.sa_stride_k + static_cast<int64_t>(mb) * BM) * (kFp32 ? 4 : 1);
          bulk_load(smem_u32(slot + kSlotRawA), ga, a_sc_bytes, full_bar(s));
          if (B_ROW) {
            const uint8_t* gb = static_cast<const uint8_t*>(p.sB) +
                                (kb * p.sb_stride_k + static_cast<int64_t>(nb) * BN) * (kFp32 ? 4 : 1);
            bulk_load(smem_u32(slot + kSlotRawB), gb, b_sc_bytes, full_bar(s));
          }
        }
      }
      // teardown: every copy this thread issued has landed before the CTA exits
      const uint32_t total = it;
      for (uint32_t j = (total > STAGES ? total - STAGES : 0); j < total; ++j)
        mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1, guard, kTimeoutTeardown);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t idesc = kFp32 ? idesc_f8(BM, BN, !B_KMAJOR) : idesc_mxf8(BM, BN, !B_KMAJOR);
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
        if (!kFp32) {
          if (!mbar_wait(tempty_bar(0), (tcount & 1) ^ 1, guard, kTimeoutMma)) { ok = false; break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          uint32_t d = tmem_base;
          if (kFp32) {
            const uint32_t b = it & 1;
            if (!mbar_wait(tempty_bar(b), ((it >> 1) & 1) ^ 1, guard, kTimeoutMma)) { ok = false; break; }
            if (!mbar_wait(full_bar(s), ph, guard, kTimeoutMma)) { ok = false; break; }
            d = tmem_base + b * 256;
          } else {
            if (!mbar_wait(full_bar(s), ph, guard, kTimeoutMma)) { ok = false; break; }
            if (!mbar_wait(sfready_bar(s), ph, guard, kTimeoutMma)) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + kOffA + s * kTileABytes);
          const uint32_t sb = smem_u32(smem + kOffB + s * kTileBBytes);
          const uint32_t sf_a = tmem_base + kTmemSf + 16 * s;
          const uint32_t sf_b = sf_a + 8;
          if (!kFp32) {
            const uint32_t tm = smem_u32(smem + kOffSlot + s * kSlotBytes + kSlotTm);
            tc_cp_32x128b_warpx4(sf_a, smem_desc(tm, 0, 128, kLayoutNone));
            tc_cp_32x128b_warpx4(sf_b, smem_desc(tm + 512, 0, 128, kLayoutNone));
            tc_cp_32x128b_warpx4(sf_b + 4, smem_desc(tm + 1024, 0, 128, kLayoutNone));
          }
#pragma unroll
          for (int k4 = 0; k4 < BK / 32; ++k4) {
            const uint64_t adesc = smem_desc(sa + 32 * k4, 16, 1024, kLayoutSw128);
            const uint64_t bdesc = B_KMAJOR ? smem_desc(sb + 32 * k4, 16, 1024, kLayoutSw128)
                                            : smem_desc(sb + 4096 * k4, kTileBBytes / 2, 1024, kLayoutSw128);
            if (kFp32)
              mma_f8(d, adesc, bdesc, idesc, k4 > 0 ? 1u : 0u);
            else
              mma_mxf8(d, adesc, bdesc, idesc, sf_a, sf_b, (kb > 0 || k4 > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
          if (kFp32) tc_commit(tfull_bar(it & 1));
        }
        if (!ok) break;
        if (!kFp32) tc_commit(tfull_bar(0));
      }
      // teardown: all MMAs this thread issued have completed
      tc_commit(final_bar);
      mbar_wait(final_bar, 0, guard, kTimeoutTeardown);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------- scale staging
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, mb, nb);
      uint32_t cur0 = 0, cur1 = 0, nxt0 = 0, nxt1 = 0;
      if (!B_ROW) {
        load_block_scales(p, nb, 0, kFp32, cur0, cur1);
        load_block_scales(p, nb, 32, kFp32, nxt0, nxt1);
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!B_ROW && kb > 0 && (kb & 31) == 0) {
          cur0 = nxt0;
          cur1 = nxt1;
          load_block_scales(p, nb, kb + 32, kFp32, nxt0, nxt1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kTimeoutScale))) { ok = false; break; }
        uint8_t* slot = smem + kOffSlot + s * kSlotBytes;
        uint32_t b0 = 0, b1 = 0;
        if (!B_ROW) {
          b0 = __shfl_sync(0xffffffffu, cur0, kb & 31);
          b1 = __shfl_sync(0xffffffffu, cur1, kb & 31);
        }
        if (kFp32) {
          if (!B_ROW && lane == 0) {
            reinterpret_cast<uint32_t*>(slot + kSlotBlk)[0] = b0;
            reinterpret_cast<uint32_t*>(slot + kSlotBlk)[1] = b1;
          }
        } else {
          // tensor-memory image of 128 scales: 32 rows of 16 B; row l holds the
          // scales of rows l, 32+l, 64+l, 96+l (one per 32-bit column), each
          // byte replicated 4x so every scale-byte selector reads the same value.
          const uint8_t* ra = slot + kSlotRawA;
          uint4 wa;
          wa.x = static_cast<uint32_t>(ra[lane]) * 0x01010101u;
          wa.y = static_cast<uint32_t>(ra[32 + lane]) * 0x01010101u;
          wa.z = static_cast<uint32_t>(ra[64 + lane]) * 0x01010101u;
          wa.w = static_cast<uint32_t>(ra[96 + lane]) * 0x01010101u;
          *reinterpret_cast<uint4*>(slot + kSlotTm + 16 * lane) = wa;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 wb;
            if (B_ROW) {
              const uint8_t* rb = slot + kSlotRawB + 128 * h;
              wb.x = static_cast<uint32_t>(rb[lane]) * 0x01010101u;
              wb.y = static_cast<uint32_t>(rb[32 + lane]) * 0x01010101u;
              wb.z = static_cast<uint32_t>(rb[64 + lane]) * 0x01010101u;
              wb.w = static_cast<uint32_t>(rb[96 + lane]) * 0x01010101u;
            } else {
              const uint32_t v = (h == 0 ? b0 : b1) * 0x01010101u;
              wb = make_uint4(v, v, v, v);
            }
            *reinterpret_cast<uint4*>(slot + kSlotTm + 512 + 512 * h + 16 * lane) = wb;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sfready_bar(s));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;   // 0..7
    const int quarter = warp & 3;      // TMEM lane quarter this warp may access
    const int half = ew >> 2;          // column half of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int row_in_tile = 32 * quarter + lane;
    uint32_t it = 0, tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, mb, nb);
      float acc[128];
      if (kFp32) {
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          const uint32_t b = it & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(b), (it >> 1) & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
          // the scale slot of this K block (written by TMA, seen through the
          // staging warp's arrival)
          if (!__all_sync(0xffffffffu, mbar_wait(sfready_bar(s), ph, guard, kTimeoutEpilogue))) { ok = false; break; }
          tc_fence_after();
          const uint8_t* slot = smem + kOffSlot + s * kSlotBytes;
          const float sa = reinterpret_cast<const float*>(slot + kSlotRawA)[row_in_tile];
          const uint32_t cbase = tmem_base + lane_addr + b * 256 + half * 128;
          if (!B_ROW) {
            const float f = sa * reinterpret_cast<const float*>(slot + kSlotBlk)[half];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(cbase + 32 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[32 * c + i] = fmaf(__uint_as_float(r[i]), f, acc[32 * c + i]);
            }
          } else {
            const float4* sbv = reinterpret_cast<const float4*>(slot + kSlotRawB) + half * 32;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(cbase + 32 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 sb = sbv[8 * c + i];
                acc[32 * c + 4 * i + 0] = fmaf(__uint_as_float(r[4 * i + 0]), sa * sb.x, acc[32 * c + 4 * i + 0]);
                acc[32 * c + 4 * i + 1] = fmaf(__uint_as_float(r[4 * i + 1]), sa * sb.y, acc[32 * c + 4 * i + 1]);
                acc[32 * c + 4 * i + 2] = fmaf(__uint_as_float(r[4 * i + 2]), sa * sb.z, acc[32 * c + 4 * i + 2]);
                acc[32 * c + 4 * i + 3] = fmaf(__uint_as_float(r[4 * i + 3]), sa * sb.w, acc[32 * c + 4 * i + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(tempty_bar(b));
            mbar_arrive(scempty_bar(s));
          }
        }
        if (!ok) break;
      } else {
        if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(0), tcount & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
        tc_fence_after();
        const uint32_t cbase = tmem_base + lane_addr + half * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(cbase + 32 * c, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * c + i] = __uint_as_float(r[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(0));
      }
      // convert to BF16 (round to nearest even) and store this thread's row
      const int64_t m = static_cast<int64_t>(mb) * BM + row_in_tile;
      const int n0 = nb * BN + half * 128;
      if (m < p.M) {
        uint16_t* drow = p.D + m * p.ldd + n0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (n0 + 8 * c < p.N) {
            uint4 o;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t packed;
              asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed) : "f"(acc[8 * c + 2 * j + 1]), "f"(acc[8 * c + 2 * j]));
              ow[j] = packed;
            }
            *reinterpret_cast<uint4*>(drow + 8 * c) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------- host --
__device__ int g_device_status;

struct DeviceInfo {
  int sms = 0;
  int* status = nullptr;
  bool attr_set[8] = {};
};

DeviceInfo g_dev[64];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

cudaError_t device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void* sym = nullptr;
    e = cudaGetSymbolAddress(&sym, g_device_status);
    if (e != cudaSuccess) return e;
    d.status = static_cast<int*>(sym);
  }
  *out = &d;
  return cudaSuccess;
}

// 2-D tensor map over a byte matrix [rows, cols] with row pitch `pitch` bytes;
// box = box_cols x box_rows; 128-byte swizzle; out-of-range reads give zeros.
bool encode_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
               uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int FMT, bool BK_, bool BR_>
cudaError_t launch_variant(const Params& prm, int grid, DeviceInfo* di, int slot, cudaStream_t stream) {
  auto kern = gemm_kernel<FMT, BK_, BR_>;
  if (!di->attr_set[slot]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    di->attr_set[slot] = true;
  }
  kern<<<grid, kThreads, kSmemAlloc, stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmProblem& pr, cudaStream_t stream, bool* unsupported) {
  *unsupported = false;
  if (pr.a.bf16 || !pr.a.k_major || !pr.a.row_groups || (pr.b.row_groups && !pr.b.k_major)) {
    *unsupported = true;
    return cudaSuccess;
  }
  DeviceInfo* di = nullptr;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;

  Params prm;
  memset(&prm, 0, sizeof(prm));
  if (!encode_2d(&prm.tmA, pr.a.data, pr.K, pr.M, pr.a.ld, BK, BM)) return cudaErrorInvalidValue;
  if (pr.b.k_major) {
    if (!encode_2d(&prm.tmB, pr.b.data, pr.K, pr.N, pr.b.ld, BK, BN)) return cudaErrorInvalidValue;
  } else {
    if (!encode_2d(&prm.tmB, pr.b.data, pr.N, pr.K, pr.b.ld, 128, BK)) return cudaErrorInvalidValue;
  }
  prm.sA = pr.a.scales;
  prm.sB = pr.b.scales;
  prm.sa_stride_k = pr.a.s_stride_k;
  prm.sb_stride_k = pr.b.s_stride_k;
  prm.sb_stride_r = pr.b.s_stride_r;
  prm.sb_len = pr.b.row_groups ? pr.b.s_stride_k : 0;
  prm.nb_blocks = (pr.N + 127) / 128;
  prm.D = static_cast<uint16_t*>(pr.d);
  prm.ldd = pr.ldd;
  prm.M = static_cast<int>(pr.M);
  prm.N = static_cast<int>(pr.N);
  prm.K = static_cast<int>(pr.K);
  prm.num_m = static_cast<int>((pr.M + BM - 1) / BM);
  prm.num_n = static_cast<int>((pr.N + BN - 1) / BN);
  prm.num_tiles = prm.num_m * prm.num_n;
  prm.num_kb = static_cast<int>(pr.K / BK);
  prm.status = di->status;
  prm.limit_ns = 2000000000ull;  // 2 s per wait
  const int grid = prm.num_tiles < di->sms ? prm.num_tiles : di->sms;

  const bool fp32 = pr.fmt == kFmtFp32;
  const bool bk = pr.b.k_major;
  const bool br = pr.b.row_groups;
  if (fp32) {
    if (bk && !br) return launch_variant<kFmtFp32, true, false>(prm, grid, di, 0, stream);
    if (!bk && !br) return launch_variant<kFmtFp32, false, false>(prm, grid, di, 1, stream);
    return launch_variant<kFmtFp32, true, true>(prm, grid, di, 2, stream);
  }
  if (bk && !br) return launch_variant<kFmtUe8m0, true, false>(prm, grid, di, 3, stream);
  if (!bk && !br) return launch_variant<kFmtUe8m0, false, false>(prm, grid, di, 4, stream);
  return launch_variant<kFmtUe8m0, true, true>(prm, grid, di, 5, stream);
}

cudaError_t read_and_clear_device_status(cudaStream_t stream, int* status) {
  *status = 0;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  DeviceInfo* di = nullptr;
  e = device_info(&di);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpy(&v, di->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpy(di->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return e;
  }
  *status = v;
  return cudaSuccess;
}

}  // namespace fp8bq
