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
// Two kernels.  gemm_pair_kernel (below; every M > 128, i.e. every shape of
// the layer) runs CTA pairs (tcgen05 cta_group::2) over 256 x 256 tiles with
// a 5-stage ring, UE8M0 scales packed four K blocks to a tensor-memory word,
// a grouped raster and split last rounds.  gemm_kernel, for M <= 128, is the
// single-CTA form described here.
//
// Kernel shape (one CTA per SM, persistent over 128 x 256 output tiles,
// 12 warps):
//   warp 0      TMA producer: A and B K-block tiles (128-byte swizzle) and the
//               raw scale vectors of each K block, into a 3-stage ring.
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma.
//   warp 2      scale staging: writes the 128x128-block scale of B into the
//               ring (FP32 path) or rearranges the UE8M0 scales into the
//               layout tcgen05.cp copies into tensor memory (block-scaled path).
//   warp 3      spare (keeps the four control warps one per sub-partition).
//   warps 4-11  epilogue; each owns 32 rows (its TMEM lane quarter) x 128
//               columns of the tile and its own 8 KB staging buffer, written
//               in the 128-byte-swizzled layout of a TMA store box.
// FP32 scales ("promotion" path): each K block's MMAs write a fresh partial
// product into one of two 256-column TMEM buffers; the epilogue warps load it,
// multiply by sA * sB and add it into FP32 register accumulators (packed
// two-wide FMAs) while the tensor core fills the other buffer.  UE8M0 scales:
// the block-scaled MMA (kind::mxf8f6f4.block_scale) applies the power-of-two
// scales itself and accumulates the whole K extent in one TMEM buffer; the
// epilogue drains it into registers once per tile and frees it before
// converting.  Either way the BF16 tile leaves through shared memory and TMA
// stores, so the epilogue warps return to the next tile at once.
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
constexpr int STAGES = 3;
constexpr int kThreads = 384;  // 12 warps: 4 control + 8 epilogue
constexpr int kEpiWarp0 = 4;
// Registers are budgeted per SM sub-partition (warp w runs on sub-partition
// w % 4, 16K registers each): three warps per sub-partition leave 168 per
// thread, enough for the 128 FP32 accumulators of an epilogue thread plus
// one 32-column tensor-memory load.
constexpr int kEpiWarps = 8;
constexpr int kTmemCols = 512;
// M blocks per raster group (L2 reuse of B), unless Params::group_m says
// otherwise.  4 measured 1-3% faster than 8 on the gate/up GEMMs and no
// slower elsewhere (2 and 6 in between, 16 slower).
constexpr int kGroupM = 4;

constexpr uint32_t kTileABytes = BM * BK;  // 16 KB
constexpr uint32_t kTileBBytes = BN * BK;  // 32 KB
constexpr uint32_t kStageBytes = 8192;     // per epilogue warp: 2 boxes of 32 rows x 64 bf16
// per-stage scale slot
constexpr uint32_t kSlotRawA = 0;      // 128 FP32 scales (512 B) or 128 UE8M0 bytes
constexpr uint32_t kSlotRawB = 512;    // 256 FP32 scales (1 KB) or 256 UE8M0 bytes
constexpr uint32_t kSlotBlk = 1536;    // two 128x128-block scales of B (FP32 path)
constexpr uint32_t kSlotTm = 1664;     // 1536 B: tensor-memory images of the UE8M0 scales
constexpr uint32_t kSlotBytes = 3200;  // multiple of 128

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + STAGES * kTileABytes;
constexpr uint32_t kOffStage = kOffB + STAGES * kTileBBytes;
constexpr uint32_t kOffSlot = kOffStage + kEpiWarps * kStageBytes;
constexpr uint32_t kOffBar = kOffSlot + STAGES * kSlotBytes;
// barriers: full[S], empty[S], sfready[S], scempty[S], tfull[2], tempty[2], final
constexpr uint32_t kNumBars = 4 * STAGES + 5;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-B alignment
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// TMEM columns: FP32 path: partial buffers at 0 and 256.  UE8M0 path: the
// accumulator at 0..255, then per stage s the A scales at 256 + 16 s (4 cols)
// and the B scales at 256 + 16 s + 8 (8 cols).
constexpr uint32_t kTmemSf = 256;

constexpr int kTimeoutProducer = 1;
constexpr int kTimeoutMma = 2;
constexpr int kTimeoutScale = 3;
constexpr int kTimeoutEpilogue = 4;
constexpr int kTimeoutTeardown = 5;
constexpr int kTimeoutSplit = 6;

struct Params {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmD;       // BF16 output, 64 x 32 boxes, 128-byte swizzle
  CUtensorMap tmSA;      // MX only: A's 1x32 scales [K/32][lds_a] bytes, boxes 128 x 4
  CUtensorMap tmSB;      // MX only: B's 1x32 scales [K/32][lds_b] bytes, boxes 256 x 4
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
  int group_m;  // M blocks per raster group: consecutive tiles walk down a group's M blocks, then across N
  int* status;
  uint64_t limit_ns;
  // Split tiles (CTA-pair kernel, BF16 D): tiles [dp_tiles, num_tiles) are
  // shared along K by all clusters.  A tile's head piece (from K block 0)
  // keeps its partial sum; every other piece stores its FP32 partial sum
  // into the workspace slot of its cluster and raises that slot's flags; the
  // head piece adds those partials and rounds the tile to BF16 once.
  // dp_tiles == num_tiles: nothing is split.
  int dp_tiles;
  CUtensorMap tmW;  // workspace [clusters * 256][256] FP32, 32 x 32 boxes, 128-byte swizzle
  float* ws;        // one 256 x 256 partial-sum slot per cluster
  int* ws_flag;     // per slot and epilogue warp slice: 1 = partial stored (0 between calls)
  // FP32 promotion path with one operand's scales in UE8M0 (a mixed pair):
  // that operand's scale bytes are staged and decoded to the FP32 value 2^e.
  int a_u8, b_u8;
  int withhold_cluster;  // test hook: this pair never raises its split flags (-1: none)
  // L2 eviction priority of the A loads and the output stores (kHint*
  // bits): a streamed A and the output go first, so that operand tiles read
  // by several tiles stay.
  uint32_t l2_hints;
  // Clock counters (nullptr: off): every CTA adds the SM cycles (clock64) and
  // the nanoseconds (globaltimer) between its start and its end, so that
  // clk[0] / clk[1] is the SM clock in GHz the GEMM ran at.
  unsigned long long* clk;
};

// Start / end stamps of a CTA for Params::clk (thread 0 only).
struct ClockStamp {
  long long c0;
  uint64_t t0;
};
__device__ __forceinline__ ClockStamp clock_begin(const Params& p) {
  ClockStamp st{0, 0};
  if (p.clk != nullptr && threadIdx.x == 0) {
    st.c0 = clock64();
    st.t0 = global_timer_ns();
  }
  return st;
}
__device__ __forceinline__ void clock_end(const Params& p, const ClockStamp& st) {
  if (p.clk != nullptr && threadIdx.x == 0) {
    const long long c1 = clock64();
    const uint64_t t1 = global_timer_ns();
    atomicAdd(p.clk, static_cast<unsigned long long>(c1 - st.c0));
    atomicAdd(p.clk + 1, static_cast<unsigned long long>(t1 - st.t0));
  }
}

constexpr uint32_t kHintAFirst = 1, kHintDFirst = 4;

// FP32 value of a UE8M0 scale byte u (2^(u - 127)); u = 0 is the subnormal
// 2^-127.  The quantizers write u in [0, 254].
__device__ __forceinline__ uint32_t ue8m0_to_f32_bits(uint32_t u) {
  return u == 0 ? 0x00400000u : (u << 23);
}

// ----------------------------------------------------------- work units --
// A cluster's work: the tiles cl, cl + ncl, ... below dp_tiles, each whole;
// then its share of the split tiles: their K blocks laid end to end (tile by
// tile) and cut into ncl ranges of nearly equal length, range c going to
// cluster c.  A range is shorter than one tile's K extent (the split tiles
// are fewer than the clusters), so it covers parts of at most two tiles: the
// tail of one (the cluster's first unit) and the head of the next (its last
// unit).  Hence a cluster holds at most one piece that does not start at K
// block 0, and a tile's head piece is the last unit of its cluster.
struct Unit {
  int tile;  // < 0: no more work
  int kb0, kb1;
  bool split;  // covers only part of the tile's K blocks
};

__device__ __forceinline__ int64_t split_bound(const Params& p, int c, int ncl) {
  return static_cast<int64_t>(p.num_tiles - p.dp_tiles) * p.num_kb * c / ncl;
}

__device__ __forceinline__ Unit split_unit(const Params& p, int64_t g, int c, int ncl) {
  const int64_t hi = split_bound(p, c + 1, ncl);
  Unit u{-1, 0, 0, false};
  if (g >= hi) return u;
  u.tile = p.dp_tiles + static_cast<int>(g / p.num_kb);
  u.kb0 = static_cast<int>(g % p.num_kb);
  const int64_t left = hi - g;
  u.kb1 = left < p.num_kb - u.kb0 ? u.kb0 + static_cast<int>(left) : p.num_kb;
  u.split = u.kb1 - u.kb0 < p.num_kb;
  return u;
}

__device__ __forceinline__ Unit first_unit(const Params& p, int c, int ncl) {
  if (c < p.dp_tiles) return Unit{c, 0, p.num_kb, false};
  return split_unit(p, split_bound(p, c, ncl), c, ncl);
}

__device__ __forceinline__ Unit next_unit(const Params& p, const Unit& u, int c, int ncl) {
  if (u.tile < p.dp_tiles) {
    const int t = u.tile + ncl;
    if (t < p.dp_tiles) return Unit{t, 0, p.num_kb, false};
    return split_unit(p, split_bound(p, c, ncl), c, ncl);
  }
  return split_unit(p, static_cast<int64_t>(u.tile - p.dp_tiles) * p.num_kb + u.kb1, c, ncl);
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int group = tile / (group_m * num_n);
  const int first_m = group * group_m;
  const int gsz = min(group_m, num_m - first_m);
  const int r = tile - group * group_m * num_n;
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

// Epilogue of one tile for one warp: BF16 conversion of the thread's 128
// accumulators (row 32*quarter + lane, columns half*128 ...), written into
// the warp's staging buffer as two 32 x 64 boxes in the 128-byte swizzled
// layout (16-byte chunk c of row r at chunk position c ^ (r % 8)), then two
// TMA stores issued by lane 0.  Rows or columns outside D are clipped by TMA.
__device__ __forceinline__ void store_tile(const Params& p, const float2 (&acc)[64], uint8_t* stage,
                                           int lane, int m0, int n0) {
  if (lane == 0) bulk_wait_group_read0();  // the previous tile's stores have left the buffer
  __syncwarp();
  const uint32_t sbase = smem_u32(stage);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int q = 32 * j + 4 * c;  // float2 index of columns 64 j + 8 c
      const uint32_t w0 = pack_bf16x2(acc[q + 0].x, acc[q + 0].y);
      const uint32_t w1 = pack_bf16x2(acc[q + 1].x, acc[q + 1].y);
      const uint32_t w2 = pack_bf16x2(acc[q + 2].x, acc[q + 2].y);
      const uint32_t w3 = pack_bf16x2(acc[q + 3].x, acc[q + 3].y);
      st_shared_v4(sbase + 4096 * j + 128 * lane + 16 * (c ^ (lane & 7)), w0, w1, w2, w3);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int x = n0 + 64 * j;
      if (x < p.N && m0 < p.M) tma_store_2d(&p.tmD, sbase + 4096 * j, x, m0);
    }
    bulk_commit_group();
  }
}

// Same stores for NBOX 64-column boxes through a single 4 KB box buffer: each
// box waits for the previous store to have read the buffer.
template <int NBOX>
__device__ __forceinline__ void store_boxes(const Params& p, const float2 (&acc)[32 * NBOX], uint8_t* stage,
                                            int lane, int m0, int n0) {
  const uint32_t sbase = smem_u32(stage);
#pragma unroll
  for (int j = 0; j < NBOX; ++j) {
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int q = 32 * j + 4 * c;
      const uint32_t w0 = pack_bf16x2(acc[q + 0].x, acc[q + 0].y);
      const uint32_t w1 = pack_bf16x2(acc[q + 1].x, acc[q + 1].y);
      const uint32_t w2 = pack_bf16x2(acc[q + 2].x, acc[q + 2].y);
      const uint32_t w3 = pack_bf16x2(acc[q + 3].x, acc[q + 3].y);
      st_shared_v4(sbase + 128 * lane + 16 * (c ^ (lane & 7)), w0, w1, w2, w3);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int x = n0 + 64 * j;
      if (x < p.N && m0 < p.M) {
        if (p.l2_hints & kHintDFirst)
          tma_store_2d_hint(&p.tmD, sbase, x, m0, l2_policy_evict_first());
        else
          tma_store_2d(&p.tmD, sbase, x, m0);
      }
      bulk_commit_group();
    }
  }
}

// FP32 tile slice stored as is (no accumulation): a split tile's partial sum
// into the workspace, the boxes and staging of add_boxes_f32.
template <int NBOX>
__device__ __forceinline__ void store_boxes_f32(const CUtensorMap* map, const float2 (&acc)[16 * NBOX], uint8_t* stage,
                                                int lane, int m0, int n0) {
  const uint32_t sbase = smem_u32(stage);
#pragma unroll
  for (int j = 0; j < NBOX; ++j) {
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int q = 16 * j + 2 * c;
      st_shared_v4f(sbase + 128 * lane + 16 * (c ^ (lane & 7)), acc[q].x, acc[q].y, acc[q + 1].x, acc[q + 1].y);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(map, sbase, n0 + 32 * j, m0);
      bulk_commit_group();
    }
  }
}

// FP32 accumulation into D (D += tile): the 32 rows x 32 NBOX columns of a
// warp, as NBOX boxes of 32 x 32 floats (128-byte rows, 128-byte swizzle)
// through one 4 KB buffer, each added into global memory by a TMA reduce.
template <int NBOX>
__device__ __forceinline__ void add_boxes_f32(const CUtensorMap* map, int xlim, int ylim, const float2 (&acc)[16 * NBOX],
                                              uint8_t* stage, int lane, int m0, int n0) {
  const uint32_t sbase = smem_u32(stage);
#pragma unroll
  for (int j = 0; j < NBOX; ++j) {
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int q = 16 * j + 2 * c;  // float2 index of columns 32 j + 4 c
      st_shared_v4f(sbase + 128 * lane + 16 * (c ^ (lane & 7)), acc[q].x, acc[q].y, acc[q + 1].x, acc[q + 1].y);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int x = n0 + 32 * j;
      if (x < xlim && m0 < ylim) tma_reduce_add_2d(map, sbase, x, m0);
      bulk_commit_group();
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
  const ClockStamp clk0 = clock_begin(p);
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
        tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
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
    // The whole warp runs the loop, so descriptors and TMEM addresses stay
    // warp-uniform; one elected lane issues the tcgen05 instructions.
    {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t idesc = kFp32 ? idesc_f8(BM, BN, !B_KMAJOR) : idesc_mxf8(BM, BN, !B_KMAJOR);
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
        if (!kFp32) {
          if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(0), (tcount & 1) ^ 1, guard, kTimeoutMma))) { ok = false; break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          uint32_t d = tmem_base;
          if (kFp32) {
            const uint32_t b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(b), ((it >> 1) & 1) ^ 1, guard, kTimeoutMma))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
            d = tmem_base + b * 256;
          } else {
            if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, mbar_wait(sfready_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + kOffA + s * kTileABytes);
          const uint32_t sb = smem_u32(smem + kOffB + s * kTileBBytes);
          const uint32_t sf_a = tmem_base + kTmemSf + 16 * s;
          const uint32_t sf_b = sf_a + 8;
          if (elect_one()) {
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
          __syncwarp();
        }
        if (!ok) break;
        if (!kFp32 && elect_one()) tc_commit(tfull_bar(0));
        __syncwarp();
      }
      // teardown: all MMAs this warp issued have completed
      if (elect_one()) tc_commit(final_bar);
      __syncwarp();
      mbar_wait(final_bar, 0, guard, kTimeoutTeardown);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------- scale staging
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
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
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;   // 0..7
    const int quarter = warp & 3;      // TMEM lane quarter this warp may access
    const int half = ew >> 2;          // column half of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int row_in_tile = 32 * quarter + lane;
    uint8_t* stage = smem + kOffStage + ew * kStageBytes;
    uint32_t it = 0, tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
      float2 acc[64];
      if (kFp32) {
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
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
          const float2 sa2 = make_float2(sa, sa);
          float2 f2 = sa2;
          if (!B_ROW) {
            const float f = sa * reinterpret_cast<const float*>(slot + kSlotBlk)[half];
            f2 = make_float2(f, f);
          }
          if (!B_ROW) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float r[32];
              tmem_ld_32x32b_x32f(cbase + 32 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                acc[16 * c + i] = __ffma2_rn(make_float2(r[2 * i], r[2 * i + 1]), f2, acc[16 * c + i]);
            }
          } else {
            // per-column B scales: 16-column loads keep the staging small
            // enough for the 128 accumulators to stay in registers
            const float2* sbv = reinterpret_cast<const float2*>(slot + kSlotRawB) + half * 64;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float r[16];
              tmem_ld_32x32b_x16f(cbase + 16 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i)
                acc[8 * c + i] = __ffma2_rn(make_float2(r[2 * i], r[2 * i + 1]), __fmul2_rn(sa2, sbv[8 * c + i]),
                                            acc[8 * c + i]);
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
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32f(cbase + 32 * c, &acc[16 * c].x);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(0));
      }
      store_tile(p, acc, stage, lane, mb * BM + 32 * quarter, nb * BN + half * 128);
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  clock_end(p, clk0);
}

// ===================================================== CTA-pair kernel ===
// Two CTAs of a cluster share every MMA (tcgen05 cta_group::2, M = 256,
// N = 256): CTA r of the pair holds rows 128 r .. of the 256-row A block, B
// rows 128 r .. of the 256-row B block, and accumulator rows 128 r .. (all 256
// columns) in its own TMEM.  Per K block each CTA loads 32 KB instead of the
// 48 KB of a 128 x 256 tile, so four stages fit beside the epilogue staging
// and the loads the tensor core waits on are a third smaller.  Roles per CTA
// are those of the single-CTA kernel; only the even-ranked (leader) CTA's MMA
// thread issues MMAs.  Barriers:
//   full[s]    leader; operand bytes of both CTAs (their TMA loads complete
//              on the leader's barrier), one arrival from the leader's producer
//              and, UE8M0 path, one from each CTA's scale staging warp once
//              its tensor-memory scale image is written
//   fullsc[s]  local; this CTA's scale vectors
//   empty[s]   local; arrived by the leader's commit, multicast to both CTAs
//   sfready[s] local; this CTA's scale staging warp (FP32 promotion path)
//   scempty[s] local; this CTA's epilogue warps (scale slot free)
//   tfull[b]   local; leader's commit, multicast
//   tempty[b]  leader; the epilogue warps of both CTAs
// Remote arrivals and waits use the default (CTA-scope) semantics: the
// barrier phases themselves order the tcgen05 / TMA traffic they guard, and
// cluster-scope releases or whole-proxy fences cost about a microsecond each.
namespace pairk {
constexpr int P_BMC = 128;   // accumulator rows per CTA
constexpr int P_BN = 256;    // tile columns
constexpr int P_BNC = 128;   // B rows loaded per CTA
constexpr uint32_t P_kTileA = P_BMC * BK;  // 16 KB
constexpr uint32_t P_kTileB = P_BNC * BK;  // 16 KB
// Register split of the FP32 promotion variant (setmaxnreg), per thread.
constexpr uint32_t kCtrlRegs = 40;
constexpr uint32_t kEpiRegs = 232;
static_assert(4 * kCtrlRegs + 8 * kEpiRegs <= 12 * 168, "register split within the launch allocation");
// Eight epilogue warps of 128 columns each.  (Sixteen warps of 64 columns,
// capped at 96 registers a thread, ran the FP32 promotion slower: it is bound
// by the FP32 pipe and tensor-memory reads, not by load latency.)
// Each warp stages its output through one 4 KB box (TMA stores, or TMA
// reduce for FP32 accumulation), which leaves room for five operand stages
// (measured 5-14% faster than four).  Storing the BF16 rows straight from
// registers instead, to make room for a sixth stage, ran the UE8M0 GEMMs up
// to 33% slower: a lane's row is 16 bytes a store, 32 rows apart.
template <int FMT, bool ACC>
struct Cfg {
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kCols = 256 / (kEpiWarps / 4);  // accumulator columns per epilogue warp
  static constexpr int kStages = 5;
  // scale slots: UE8M0, two groups of four K blocks; otherwise one per stage
  static constexpr int kSlots = (FMT == kFmtUe8m0) ? 2 : kStages;
  static constexpr uint32_t kStage = 4096u;  // one 32 x 64 bf16 output box per warp
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * P_kTileA;
  static constexpr uint32_t kOffStage = kOffB + kStages * P_kTileB;
  static constexpr uint32_t kOffSlot = kOffStage + kEpiWarps * kStage;
  static constexpr uint32_t kOffBar = kOffSlot + kSlots * kSlotBytes;
  // full, fullsc, empty, sfready, scempty [S]; tfull[2], tempty[2], final;
  // eload[kEpiWarps] (split-tile partial-sum loads of the epilogue warps);
  // gfull, gready, gempty [2] (UE8M0 scale-factor groups)
  static constexpr uint32_t kNumBars = 5 * kStages + 5 + kEpiWarps + 6;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kTmemSf + 16 * kStages <= kTmemCols, "scale-factor columns");
  // the split-tile head piece stages a warp's 32 x 128 FP32 partial (16 KB)
  // in the operand stages
  static_assert(kEpiWarps * 16384u <= kStages * (P_kTileA + P_kTileB), "partial-sum staging");
};
}  // namespace pairk

template <int FMT, bool B_KMAJOR, bool B_ROW, bool ACC = false>
__global__ void __launch_bounds__(pairk::Cfg<FMT, ACC>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ Params p) {
  // ACC: D is FP32 and the tile is added into it (D += A B^T), else BF16 D = A B^T
  using pairk::P_BMC;
  using pairk::P_BN;
  using pairk::P_BNC;
  using pairk::P_kTileA;
  using pairk::P_kTileB;
  using C = pairk::Cfg<FMT, ACC>;
  constexpr int P_STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool kFp32 = (FMT == kFmtFp32);
  constexpr bool kMx = (FMT == kFmtMx);  // 1x32 scales: four per 128-long K block
  // UE8M0 with 1x128 groups or 128x128 blocks: one scale byte per row and K
  // block, so the four bytes of a tensor-memory scale word hold four K
  // blocks' scales (a group) and are copied in once per group; each MMA
  // selects its K block's byte through the scale-factor IDs
  constexpr bool kPack = (FMT == kFmtUe8m0);
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto full_bar = [&](int s) { return bar(s); };
  auto fullsc_bar = [&](int s) { return bar(P_STAGES + s); };
  auto empty_bar = [&](int s) { return bar(2 * P_STAGES + s); };
  auto sfready_bar = [&](int s) { return bar(3 * P_STAGES + s); };
  auto scempty_bar = [&](int s) { return bar(4 * P_STAGES + s); };
  // accumulator buffers: UE8M0 / MX one (0); FP32 two 256-column partial
  // buffers, one per K-block parity
  auto tfull_bar = [&](int b) { return bar(5 * P_STAGES + b); };
  auto tempty_bar = [&](int b) { return bar(5 * P_STAGES + 2 + b); };
  const uint32_t final_bar = bar(5 * P_STAGES + 4);
  auto eload_bar = [&](int w) { return bar(5 * P_STAGES + 5 + w); };
  auto gfull_bar = [&](int g) { return bar(5 * P_STAGES + 5 + C::kEpiWarps + g); };   // a group's raw scales landed
  auto gready_bar = [&](int g) { return bar(5 * P_STAGES + 7 + C::kEpiWarps + g); };  // its scale words staged (leader)
  auto gempty_bar = [&](int g) { return bar(5 * P_STAGES + 9 + C::kEpiWarps + g); };  // its copies and MMAs done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const WaitGuard guard{abort_flag, p.status, p.limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      // UE8M0: the scale-staging warps of both CTAs also arrive on full[s]
      // (MX: two staging warps per CTA, one for A's scales, one for B's)
      mbar_init(full_bar(s), kMx ? 5 : 1);
      mbar_init(fullsc_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sfready_bar(s), 1);
      mbar_init(scempty_bar(s), C::kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * C::kEpiWarps);  // every epilogue warp of both CTAs drains it
    }
    mbar_init(final_bar, 1);
    for (int w = 0; w < C::kEpiWarps; ++w) mbar_init(eload_bar(w), 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(gfull_bar(g), 1);
      mbar_init(gready_bar(g), 2);  // the staging warps of both CTAs
      mbar_init(gempty_bar(g), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialized, TMEM of both allocated
  tc_fence_after();
  const ClockStamp clk0 = clock_begin(p);
  const uint32_t tmem_base = *tmem_holder;
  const int cl = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(nclusters_x());
  // FP32 promotion: the epilogue holds 128 FP32 accumulators and two
  // 32-column partial chunks per thread, so the control warpgroup (warps
  // 0-3) hands registers over to the two epilogue warpgroups: 4 warps x 40
  // plus 8 warps x 232 is exactly the 12 x 168 the CTA was launched with.
  // Each role sets its budget at its own entry, so the compiler allots each
  // role's code its own register count (the bounded waits are inlined for
  // the same reason: an out-of-line callee cannot serve both budgets).
  auto ctrl_regs = [&]() {
    if constexpr (kFp32) regs_dealloc<pairk::kCtrlRegs>();
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Warp-uniform loop; one elected lane issues the copies.
    ctrl_regs();
    prefetch_tensormap(&p.tmA);
    prefetch_tensormap(&p.tmB);
    const uint64_t pol_a = (p.l2_hints & kHintAFirst) ? l2_policy_evict_first() : 0;
    if (kMx || kPack) {
      prefetch_tensormap(&p.tmSA);
      if (kMx || B_ROW) prefetch_tensormap(&p.tmSB);
    }
    uint32_t it = 0, gi = 0;
    bool ok = true;
    for (Unit u = first_unit(p, cl, ncl); ok && u.tile >= 0; u = next_unit(p, u, cl, ncl)) {
      int mb, nb;
      tile_coords(u.tile, p.num_m, p.num_n, p.group_m, mb, nb);
      const int64_t row0 = static_cast<int64_t>(mb) * (2 * P_BMC) + P_BMC * rank;  // this CTA's A rows
      const int32_t brow = nb * P_BN + P_BNC * static_cast<int>(rank);
      // scale bytes per entry; a UE8M0 operand of the FP32 path lands as raw
      // bytes in the slot's staging area and is decoded by the staging warp
      const uint32_t esz_a = kFp32 && !p.a_u8 ? 4u : 1u;
      const uint32_t esz_b = kFp32 && !p.b_u8 ? 4u : 1u;
      const uint32_t dst_a = kFp32 && p.a_u8 ? kSlotTm : kSlotRawA;
      const uint32_t dst_b = kFp32 && p.b_u8 ? kSlotTm + 128 : kSlotRawB;
      const bool a_sc = row0 < p.sa_stride_k;  // rows past the padded scale rows carry only zeros
      uint32_t b_sc_bytes = 0;
      if (B_ROW) {
        const int64_t left = p.sb_len - static_cast<int64_t>(nb) * P_BN;
        b_sc_bytes = static_cast<uint32_t>(left < P_BN ? left : P_BN) * esz_b;
      }
      const uint8_t* ga = static_cast<const uint8_t*>(p.sA) + row0 * esz_a;
      const uint8_t* gb = static_cast<const uint8_t*>(p.sB) + static_cast<int64_t>(nb) * P_BN * esz_b;
      for (int kb = u.kb0; kb < u.kb1; ++kb, ++it) {
        const int s = it % P_STAGES;
        const uint32_t ph = (it / P_STAGES) & 1;
        if (kPack && (kb == u.kb0 || (kb & 3) == 0)) {
          // a new scale group (K blocks 4g .. 4g + 3): its raw scale bytes,
          // [4][128] of A and, for row-group B, [4][256] of B, as two boxes
          // into group slot gi % 2 (the first two stage slots), once the
          // group that used the slot before is done
          const int gs = static_cast<int>(gi & 1);
          if (!__all_sync(0xffffffffu, mbar_wait(gempty_bar(gs), ((gi >> 1) & 1) ^ 1, guard, kTimeoutProducer))) {
            ok = false;
            break;
          }
          if (elect_one()) {
            uint8_t* gslot = smem + C::kOffSlot + gs * kSlotBytes;
            mbar_arrive_expect_tx(gfull_bar(gs), 4u * 128u + (B_ROW ? 4u * 256u : 0u));
            tma_load_2d(smem_u32(gslot + kSlotRawA), &p.tmSA, gfull_bar(gs), static_cast<int32_t>(row0), kb & ~3);
            if (B_ROW) tma_load_2d(smem_u32(gslot + kSlotRawB), &p.tmSB, gfull_bar(gs), nb * P_BN, kb & ~3);
          }
          __syncwarp();
          ++gi;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(empty_bar(s), ph ^ 1, guard, kTimeoutProducer))) { ok = false; break; }
        if (kFp32 && !__all_sync(0xffffffffu, mbar_wait(scempty_bar(s), ph ^ 1, guard, kTimeoutProducer))) { ok = false; break; }
        if (elect_one()) {
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * (P_kTileA + P_kTileB));
          const uint32_t fb = mapa_shared(full_bar(s), 0);
          const uint32_t sa = smem_u32(smem + C::kOffA + s * P_kTileA);
          const uint32_t sb = smem_u32(smem + C::kOffB + s * P_kTileB);
          if (pol_a != 0)
            tma_load_2d_pair_hint(sa, &p.tmA, fb, kb * BK, static_cast<int32_t>(row0), pol_a);
          else
            tma_load_2d_pair(sa, &p.tmA, fb, kb * BK, static_cast<int32_t>(row0));
          const int32_t bc0 = B_KMAJOR ? kb * BK : brow, bc1 = B_KMAJOR ? brow : kb * BK;
          tma_load_2d_pair(sb, &p.tmB, fb, bc0, bc1);
          // this CTA's scale vectors (its own 128 A rows; all 256 B columns)
          uint8_t* slot = smem + C::kOffSlot + s * kSlotBytes;
          if (kPack) {
            // the scales travel per group (above)
          } else if (kMx) {
            // the K block's four 1x32 scale rows of A (128 rows) and of B (256
            // rows) as two 2-D boxes; past-the-end rows read as zeros
            mbar_arrive_expect_tx(fullsc_bar(s), 4u * 128u + 4u * 256u);
            tma_load_2d(smem_u32(slot + kSlotRawA), &p.tmSA, fullsc_bar(s), static_cast<int32_t>(row0), 4 * kb);
            tma_load_2d(smem_u32(slot + kSlotRawB), &p.tmSB, fullsc_bar(s), nb * P_BN, 4 * kb);
          } else {
            mbar_arrive_expect_tx(fullsc_bar(s), (a_sc ? 128u * esz_a : 0u) + b_sc_bytes);
            if (a_sc) bulk_load(smem_u32(slot + dst_a), ga + kb * p.sa_stride_k * esz_a, 128u * esz_a, fullsc_bar(s));
            if (B_ROW) bulk_load(smem_u32(slot + dst_b), gb + kb * p.sb_stride_k * esz_b, b_sc_bytes, fullsc_bar(s));
          }
        }
        __syncwarp();
      }
    }
    // teardown: every stage this CTA loaded has been consumed (so its copies
    // landed) before the CTA exits
    const uint32_t total = it;
    for (uint32_t j = (total > P_STAGES ? total - P_STAGES : 0); j < total; ++j) {
      mbar_wait(empty_bar(j % P_STAGES), (j / P_STAGES) & 1, guard, kTimeoutTeardown);
      if (!kPack) mbar_wait(fullsc_bar(j % P_STAGES), (j / P_STAGES) & 1, guard, kTimeoutTeardown);
    }
    // (a group's scale boxes have landed once its MMAs ran: the empty
    // barriers above come after them)
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // The whole warp runs the loop, so descriptors and TMEM addresses stay
    // warp-uniform; one elected lane issues the tcgen05 instructions.
    ctrl_regs();
    if (leader) {
      uint32_t it = 0, tcount = 0, gi = 0;
      int gs_cur = 0;  // UE8M0: the scale group slot of the K block at hand
      bool ok = true;
      const uint32_t idesc = kFp32 ? idesc_f8(2 * P_BMC, P_BN, !B_KMAJOR) : idesc_mxf8(2 * P_BMC, P_BN, !B_KMAJOR);
      for (Unit u = first_unit(p, cl, ncl); ok && u.tile >= 0; u = next_unit(p, u, cl, ncl), ++tcount) {
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++it) {
          const int s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          const uint32_t d = tmem_base;
          if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + C::kOffA + s * P_kTileA);
          const uint32_t sb = smem_u32(smem + C::kOffB + s * P_kTileB);
          if constexpr (kFp32) {
            // Promotion: K block kb writes a fresh partial (accumulate off at
            // its first MMA) into the 256-column buffer of its parity, once
            // the epilogue has drained that buffer's previous partial.  (Two
            // N = 128 halves per K block, each on its own barrier, were
            // measured slower: each tcgen05.mma costs the issuing warp tens
            // of cycles, and eight of them per K block outran the 512
            // cycles of tensor work.)
            const uint32_t pb = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(pb), ((it >> 1) & 1) ^ 1, guard, kTimeoutMma))) {
              ok = false;
            } else {
              tc_fence_after();
              if (elect_one()) {
                const uint32_t dq = d + pb * 256;
#pragma unroll
                for (int k4 = 0; k4 < BK / 32; ++k4) {
                  const uint64_t adesc = smem_desc(sa + 32 * k4, 16, 1024, kLayoutSw128);
                  const uint64_t bdesc = B_KMAJOR ? smem_desc(sb + 32 * k4, 16, 1024, kLayoutSw128)
                                                  : smem_desc(sb + 4096 * k4, P_kTileB, 1024, kLayoutSw128);
                  mma_f8_pair(dq, adesc, bdesc, idesc, k4 > 0 ? 1u : 0u);
                }
                tc_commit_pair(empty_bar(s), 0x3);
                tc_commit_pair(tfull_bar(pb), 0x3);
              }
              __syncwarp();
            }
            if (!ok) break;
          } else {
          // scale-factor columns: MX, per stage; UE8M0, per scale group slot
          const bool group_start = kPack && (kb == u.kb0 || (kb & 3) == 0);
          if (group_start) {
            gs_cur = static_cast<int>(gi & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(gready_bar(gs_cur), (gi >> 1) & 1, guard, kTimeoutMma))) {
              ok = false;
              break;
            }
            tc_fence_after();
            ++gi;
          }
          const uint32_t sf_a = tmem_base + kTmemSf + 16 * (kPack ? gs_cur : s);
          const uint32_t sf_b = sf_a + 8;
          auto issue_sf = [&]() {
            const uint32_t tm = smem_u32(smem + C::kOffSlot + (kPack ? gs_cur : s) * kSlotBytes + kSlotTm);
            tc_cp_32x128b_warpx4_pair(sf_a, smem_desc(tm, 0, 128, kLayoutNone));
            tc_cp_32x128b_warpx4_pair(sf_b, smem_desc(tm + 512, 0, 128, kLayoutNone));
            tc_cp_32x128b_warpx4_pair(sf_b + 4, smem_desc(tm + 1024, 0, 128, kLayoutNone));
          };
          auto issue_mma = [&]() {
#pragma unroll
            for (int k4 = 0; k4 < BK / 32; ++k4) {
              const uint64_t adesc = smem_desc(sa + 32 * k4, 16, 1024, kLayoutSw128);
              const uint64_t bdesc = B_KMAJOR ? smem_desc(sb + 32 * k4, 16, 1024, kLayoutSw128)
                                              : smem_desc(sb + 4096 * k4, P_kTileB, 1024, kLayoutSw128);
              // scale-factor IDs (A at bits 29-30, B at bits 4-5) select the
              // byte of each scale word: MX, sub-block k4's scale; UE8M0,
              // K block kb's scale within its group
              const uint32_t sel = kMx ? static_cast<uint32_t>(k4) : static_cast<uint32_t>(kb & 3);
              const uint32_t idk = idesc | (sel << 29) | (sel << 4);
              mma_mxf8_pair(d, adesc, bdesc, idk, sf_a, sf_b, (kb > u.kb0 || k4 > 0) ? 1u : 0u);
            }
            tc_commit_pair(empty_bar(s), 0x3);
            // the group's last K block: its scale words (smem and TMEM) are
            // free once these MMAs are done
            if (kPack && ((kb & 3) == 3 || kb == u.kb1 - 1)) tc_commit_pair(gempty_bar(gs_cur), 0x3);
          };
          const bool copy_sf = !kPack || group_start;
          if (kb == u.kb0) {
            // first K block of a tile (or piece): the scale factors (own TMEM columns)
            // are copied while the epilogue still drains the accumulator of
            // the previous tile; the MMAs wait for it
            if (elect_one()) issue_sf();
            __syncwarp();
            if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(0), (tcount & 1) ^ 1, guard, kTimeoutMma))) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) issue_mma();
          } else if (elect_one()) {
            if (copy_sf) issue_sf();
            issue_mma();
          }
          __syncwarp();
          }
        }
        if (!ok) break;
        if (!kFp32 && elect_one()) tc_commit_pair(tfull_bar(0), 0x3);
        __syncwarp();
      }
      if (elect_one()) tc_commit_pair(final_bar, 0x1);
      __syncwarp();
      mbar_wait(final_bar, 0, guard, kTimeoutTeardown);
    }
  } else if (warp == 2 || (kMx && warp == 3)) {
    // ------------------------------------------------------- scale staging
    // MX: warp 2 stages A's scale words, warp 3 B's (four bytes each).
    ctrl_regs();
    const bool stage_a = !kMx || warp == 2;
    const bool stage_b = !kMx || warp == 3;
    uint32_t it = 0, gi = 0;
    bool ok = true;
    const uint32_t full_leader_base = mapa_shared(full_bar(0), 0);
    const uint32_t gready_leader_base = mapa_shared(gready_bar(0), 0);
    for (Unit u = first_unit(p, cl, ncl); ok && u.tile >= 0; u = next_unit(p, u, cl, ncl)) {
      int mb, nb;
      tile_coords(u.tile, p.num_m, p.num_n, p.group_m, mb, nb);
      uint32_t cur0 = 0, cur1 = 0, nxt0 = 0, nxt1 = 0;
      const bool sb_fp32 = kFp32 && !p.b_u8;  // B's block scales stored as FP32
      if (!B_ROW) {
        // lane l holds K block (kb0 rounded down to 32) + l, then the next 32
        const int base = u.kb0 & ~31;
        load_block_scales(p, nb, base, sb_fp32, cur0, cur1);
        load_block_scales(p, nb, base + 32, sb_fp32, nxt0, nxt1);
      }
      for (int kb = u.kb0; kb < u.kb1; ++kb, ++it) {
        const int s = it % P_STAGES;
        const uint32_t ph = (it / P_STAGES) & 1;
        if (!B_ROW && kb > u.kb0 && (kb & 31) == 0) {
          cur0 = nxt0;
          cur1 = nxt1;
          load_block_scales(p, nb, kb + 32, sb_fp32, nxt0, nxt1);
        }
        if constexpr (kPack) {
          // UE8M0: the scale words of a group (K blocks 4g .. 4g + 3), byte j
          // of a row's word the row's scale in K block 4g + j, staged once
          // per group into its slot when its raw bytes have landed
          if (kb != u.kb0 && (kb & 3) != 0) continue;
          const int gs = static_cast<int>(gi & 1);
          if (!__all_sync(0xffffffffu, mbar_wait(gfull_bar(gs), (gi >> 1) & 1, guard, kTimeoutScale))) {
            ok = false;
            break;
          }
          ++gi;
          uint8_t* gslot = smem + C::kOffSlot + gs * kSlotBytes;
          auto pack4 = [&](const uint8_t* raw, int stride, int i) -> uint32_t {
            return static_cast<uint32_t>(raw[i]) | (static_cast<uint32_t>(raw[stride + i]) << 8) |
                   (static_cast<uint32_t>(raw[2 * stride + i]) << 16) | (static_cast<uint32_t>(raw[3 * stride + i]) << 24);
          };
          const uint8_t* ra = gslot + kSlotRawA;
          *reinterpret_cast<uint4*>(gslot + kSlotTm + 16 * lane) =
              make_uint4(pack4(ra, 128, lane), pack4(ra, 128, 32 + lane), pack4(ra, 128, 64 + lane), pack4(ra, 128, 96 + lane));
          uint32_t blk[2] = {0, 0};
          if (!B_ROW) {
            // the two 128x128 blocks' scales of the group's four K blocks
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int kj = ((kb & ~3) + j) & 31;
              blk[0] |= (__shfl_sync(0xffffffffu, cur0, kj) & 0xFFu) << (8 * j);
              blk[1] |= (__shfl_sync(0xffffffffu, cur1, kj) & 0xFFu) << (8 * j);
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 wb;
            if (B_ROW) {
              const uint8_t* rb = gslot + kSlotRawB + 128 * h;
              wb = make_uint4(pack4(rb, 256, lane), pack4(rb, 256, 32 + lane), pack4(rb, 256, 64 + lane),
                              pack4(rb, 256, 96 + lane));
            } else {
              wb = make_uint4(blk[h], blk[h], blk[h], blk[h]);
            }
            *reinterpret_cast<uint4*>(gslot + kSlotTm + 512 + 512 * h + 16 * lane) = wb;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(gready_leader_base + 8 * gs);
          continue;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(fullsc_bar(s), ph, guard, kTimeoutScale))) { ok = false; break; }
        uint8_t* slot = smem + C::kOffSlot + s * kSlotBytes;
        uint32_t b0 = 0, b1 = 0;
        if (!B_ROW) {
          b0 = __shfl_sync(0xffffffffu, cur0, kb & 31);
          b1 = __shfl_sync(0xffffffffu, cur1, kb & 31);
        }
        if (kFp32) {
          if (!B_ROW && lane == 0) {
            reinterpret_cast<uint32_t*>(slot + kSlotBlk)[0] = p.b_u8 ? ue8m0_to_f32_bits(b0) : b0;
            reinterpret_cast<uint32_t*>(slot + kSlotBlk)[1] = p.b_u8 ? ue8m0_to_f32_bits(b1) : b1;
          }
          // a mixed pair: the UE8M0 operand's raw scale bytes, decoded into
          // the FP32 scale vectors the epilogue reads
          if (p.a_u8) {
            const uint8_t* raw = slot + kSlotTm;
            uint32_t* f = reinterpret_cast<uint32_t*>(slot + kSlotRawA);
#pragma unroll
            for (int j = 0; j < 4; ++j) f[32 * j + lane] = ue8m0_to_f32_bits(raw[32 * j + lane]);
          }
          if (B_ROW && p.b_u8) {
            const uint8_t* raw = slot + kSlotTm + 128;
            uint32_t* f = reinterpret_cast<uint32_t*>(slot + kSlotRawB);
#pragma unroll
            for (int j = 0; j < 8; ++j) f[32 * j + lane] = ue8m0_to_f32_bits(raw[32 * j + lane]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(sfready_bar(s));
        } else {
          // a row's scale word: the one scale replicated (1x128 groups, any
          // byte selects it), or MX: the four sub-block scales, byte t = t-th
          auto word = [&](const uint8_t* raw, int stride, int i) -> uint32_t {
            if (!kMx) return static_cast<uint32_t>(raw[i]) * 0x01010101u;
            return static_cast<uint32_t>(raw[i]) | (static_cast<uint32_t>(raw[stride + i]) << 8) |
                   (static_cast<uint32_t>(raw[2 * stride + i]) << 16) | (static_cast<uint32_t>(raw[3 * stride + i]) << 24);
          };
          if (stage_a) {
            const uint8_t* ra = slot + kSlotRawA;
            uint4 wa;
            wa.x = word(ra, 128, lane);
            wa.y = word(ra, 128, 32 + lane);
            wa.z = word(ra, 128, 64 + lane);
            wa.w = word(ra, 128, 96 + lane);
            *reinterpret_cast<uint4*>(slot + kSlotTm + 16 * lane) = wa;
          }
#pragma unroll
          for (int h = 0; h < 2 && stage_b; ++h) {
            uint4 wb;
            if (B_ROW) {
              const uint8_t* rb = slot + kSlotRawB + 128 * h;
              wb.x = word(rb, 256, lane);
              wb.y = word(rb, 256, 32 + lane);
              wb.z = word(rb, 256, 64 + lane);
              wb.w = word(rb, 256, 96 + lane);
            } else {
              const uint32_t v = (h == 0 ? b0 : b1) * 0x01010101u;
              wb = make_uint4(v, v, v, v);
            }
            *reinterpret_cast<uint4*>(slot + kSlotTm + 512 + 512 * h + 16 * lane) = wb;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(full_leader_base + 8 * s);
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lanes 32 (w % 4) .. and a slice of kCols columns.
    if constexpr (kFp32) regs_alloc<pairk::kEpiRegs>();
    constexpr int kCols = C::kCols;
    constexpr int kAcc = kCols / 2;
    const int ew = warp - kEpiWarp0;
    const int quarter = warp & 3;
    const int slice = ew >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int row_in_tile = 32 * quarter + lane;
    uint8_t* stage = smem + C::kOffStage + ew * C::kStage;
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    uint32_t it = 0, tcount = 0, nload = 0;
    bool ok = true;
    for (Unit u = first_unit(p, cl, ncl); ok && u.tile >= 0; u = next_unit(p, u, cl, ncl), ++tcount) {
      int mb, nb;
      tile_coords(u.tile, p.num_m, p.num_n, p.group_m, mb, nb);
      float2 acc[kAcc];
      if (kFp32) {
#pragma unroll
        for (int i = 0; i < kAcc; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++it) {
          const int s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          const uint32_t b = it & 1;  // the partial buffer of this K block's parity
          const int q = static_cast<int>(b);
          if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(q), (it >> 1) & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
          if (!__all_sync(0xffffffffu, mbar_wait(sfready_bar(s), ph, guard, kTimeoutEpilogue))) { ok = false; break; }
          tc_fence_after();
          const uint8_t* slot = smem + C::kOffSlot + s * kSlotBytes;
          const float sa = reinterpret_cast<const float*>(slot + kSlotRawA)[row_in_tile];
          const uint32_t cbase = tmem_base + lane_addr + b * 256 + slice * kCols;
          const float2 sa2 = make_float2(sa, sa);
          // The warp's 128 columns are tile columns 128 slice .. + 127, one
          // 128x128 block of B.  Two 32-column chunks are in flight: chunk
          // c + 1 loads while chunk c is promoted, so each load's latency
          // hides behind multiply-adds.
          static_assert(kCols == 128, "four 32-column chunks per warp");
          float ra[32], rb[32];
          float2 f2 = sa2;
          if (!B_ROW) {
            const float f = sa * reinterpret_cast<const float*>(slot + kSlotBlk)[slice];
            f2 = make_float2(f, f);
          }
          const float2* sbv = reinterpret_cast<const float2*>(slot + kSlotRawB) + slice * kAcc;
          auto promote = [&](const float* r, int c) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              // per-column B scales (row groups) or the block's one factor
              const float2 g = B_ROW ? __fmul2_rn(sa2, sbv[16 * c + i]) : f2;
              acc[16 * c + i] = __ffma2_rn(make_float2(r[2 * i], r[2 * i + 1]), g, acc[16 * c + i]);
            }
          };
          tmem_ld_32x32b_x32f(cbase, ra);
          tmem_wait_ld_regs32(ra);
          tmem_ld_32x32b_x32f(cbase + 32, rb);
          promote(ra, 0);
          tmem_wait_ld_regs32(rb);
          tmem_ld_32x32b_x32f(cbase + 64, ra);
          promote(rb, 1);
          tmem_wait_ld_regs32(ra);
          tmem_ld_32x32b_x32f(cbase + 96, rb);
          promote(ra, 2);
          tmem_wait_ld_regs32(rb);
          // every load of the buffer has completed: hand it back to the MMA
          // before the last chunk's multiply-adds
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * q);
          promote(rb, 3);
          __syncwarp();
          if (lane == 0) mbar_arrive(scempty_bar(s));  // the scale slot's last read (per-column scales) is done
        }
        if (!ok) break;
      } else {
        if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(0), tcount & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
        tc_fence_after();
        const uint32_t cbase = tmem_base + lane_addr + slice * kCols;
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld_32x32b_x32f(cbase + 32 * c, &acc[16 * c].x);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader0);
      }
      const int m0 = mb * (2 * P_BMC) + P_BMC * static_cast<int>(rank) + 32 * quarter;
      const int n0 = nb * P_BN + slice * kCols;  // this warp's tile columns
      if constexpr (ACC) {
        add_boxes_f32<kCols / 32>(&p.tmD, p.N, p.M, acc, stage, lane, m0, n0);
      } else {
        if (u.split) {
          const int sub = 8 * static_cast<int>(rank) + ew;  // this warp's slice of the tile
          const int wrow = P_BMC * static_cast<int>(rank) + 32 * quarter;
          // In the cluster's last unit the operand stages are idle once its
          // accumulator is complete: each epilogue warp then stages its whole
          // 32 x 128 FP32 slice (four 32 x 32 boxes) in 16 KB of them.
          const bool last = next_unit(p, u, cl, ncl).tile < 0;
          const uint32_t big = smem_u32(smem + C::kOffA + ew * 16384);
          if (u.kb0 > 0) {
            // not the head piece: partial sum into this cluster's slot, then
            // the flag (release, after the stores have been performed)
            if (last) {
#pragma unroll
              for (int j = 0; j < kCols / 32; ++j)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const int q = 16 * j + 2 * c;
                  st_shared_v4f(big + 4096 * j + 128 * lane + 16 * (c ^ (lane & 7)), acc[q].x, acc[q].y, acc[q + 1].x,
                                acc[q + 1].y);
                }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                for (int j = 0; j < kCols / 32; ++j)
                  tma_store_2d(&p.tmW, big + 4096 * j, slice * kCols + 32 * j, cl * 256 + wrow);
                bulk_commit_group();
              }
            } else {
              store_boxes_f32<kCols / 32>(&p.tmW, acc, stage, lane, cl * 256 + wrow, slice * kCols);
            }
            if (lane == 0) {
              bulk_wait_group0();
              fence_proxy_async_global();
              if (cl != p.withhold_cluster) st_release_gpu(p.ws_flag + 16 * cl + sub, 1);
            }
            __syncwarp();
            continue;
          }
          // head piece (always its cluster's last unit): add the partials of
          // the clusters whose ranges start inside this tile, in cluster
          // order, each brought in by four TMA box loads; reset their flags
          const int64_t tile_end = static_cast<int64_t>(u.tile - p.dp_tiles + 1) * p.num_kb;
          for (int c = cl + 1; c < ncl && split_bound(p, c, ncl) < tile_end; ++c) {
            int* flag = p.ws_flag + 16 * c + sub;
            bool got = true;
            if (lane == 0) {
              got = flag_wait(flag, 1, guard, kTimeoutSplit);
              if (got) {
                fence_proxy_async_global();
                mbar_arrive_expect_tx(eload_bar(ew), 4096u * (kCols / 32));
                for (int j = 0; j < kCols / 32; ++j)
                  tma_load_2d(big + 4096 * j, &p.tmW, eload_bar(ew), slice * kCols + 32 * j, c * 256 + wrow);
              }
            }
            if (!__all_sync(0xffffffffu, __shfl_sync(0xffffffffu, got, 0))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, mbar_wait(eload_bar(ew), nload & 1, guard, kTimeoutSplit))) { ok = false; break; }
            ++nload;
#pragma unroll
            for (int j = 0; j < kCols / 32; ++j)
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                const int q = 16 * j + 2 * cc;
                const float4 v = ld_shared_v4f(big + 4096 * j + 128 * lane + 16 * (cc ^ (lane & 7)));
                acc[q] = __fadd2_rn(acc[q], make_float2(v.x, v.y));
                acc[q + 1] = __fadd2_rn(acc[q + 1], make_float2(v.z, v.w));
              }
            fence_proxy_async_smem();  // these reads before the next loads into the buffer
            __syncwarp();
            if (lane == 0) *flag = 0;
          }
          if (!ok) break;
        }
        store_boxes<kCols / 64>(p, acc, stage, lane, m0, n0);
      }
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  } else {
    ctrl_regs();  // the idle warp 3 releases its registers with its warpgroup
  }

  tc_fence_before();
  cluster_sync();  // both CTAs done with TMEM, barriers and each other's smem
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  clock_end(p, clk0);
}

// ================================================ fused quantize-on-load ===
// CTA-pair kernel whose A operand arrives in BF16 [M, K] and is quantized in
// shared memory, K block by K block, with the arithmetic of the 1x128
// activation quantizer (same group, same scale, same codes).  Per stage the
// producer TMA-loads the BF16 A tile (two 64-column boxes, 128-byte swizzle)
// on a CTA-local barrier and the B tile as in the pair kernel; the eight
// epilogue warps quantize the tile (two threads per 128-long row), write the
// E4M3 codes in the MMA's swizzled K-major layout and the row scale (FP32
// ring entry, or the UE8M0 tensor-memory image), and arrive on the leader's
// `aready` barrier that the MMA thread waits on.  With FP32 scales the same
// warps alternate between quantizing K block j and promoting K block j - 1.
// A and B-block scales of the FP32 path sit in rings of kRing entries indexed
// by iteration, each with its own barrier, so no writer can run a full ring
// ahead of its reader.
namespace fusedk {
constexpr int F_STAGES = 2;
constexpr int kRing = 4;
constexpr uint32_t F_kTileAbf = 128 * 128 * 2;  // two 16 KB boxes of 64 bf16 columns
constexpr uint32_t F_kTileA = 128 * 128;
constexpr uint32_t F_kTileB = 128 * 128;
constexpr uint32_t F_kOffAbf = 0;
constexpr uint32_t F_kOffA = F_kOffAbf + F_STAGES * F_kTileAbf;
constexpr uint32_t F_kOffB = F_kOffA + F_STAGES * F_kTileA;
constexpr uint32_t F_kOffStage = F_kOffB + F_STAGES * F_kTileB;
constexpr uint32_t F_kOffSlot = F_kOffStage + kEpiWarps * kStageBytes;  // per stage: raw B scales, SF images
constexpr uint32_t F_kOffRing = F_kOffSlot + F_STAGES * kSlotBytes;     // kRing x (128 A scales + 2 B scales)
constexpr uint32_t F_kRingBytes = 512 + 16;
constexpr uint32_t F_kOffBar = F_kOffRing + kRing * F_kRingBytes;
// full, fullsc, empty, sfmma, aready [S]; aconv, sfready [kRing]; tfull[2], tempty[2], final
constexpr uint32_t F_kNumBars = 5 * F_STAGES + 2 * kRing + 5;
constexpr uint32_t F_kOffMisc = (F_kOffBar + F_kNumBars * 8 + 15) / 16 * 16;
constexpr uint32_t F_kSmemBytes = F_kOffMisc + 16;
constexpr uint32_t F_kSmemAlloc = F_kSmemBytes + 1024;
static_assert(F_kSmemAlloc <= 232448, "shared memory budget");
}  // namespace fusedk

// Quantize one 64-column half of row r of the staged BF16 A tile.  The
// partner thread (lane ^ 1) holds the other half; the two exchange their amax.
template <int FMT>
__device__ __forceinline__ void fused_convert_half(uint32_t abf, uint32_t afp8, int r, int h, float* ring_sa,
                                                   uint8_t* sf_image) {
  const uint32_t src = abf + h * 16384 + r * 128;
  const int sw = r & 7;
  float m = 0.0f;
#pragma unroll
  for (int c = 0; c < 8; ++c) m = amax8(m, ld_shared_v4(src + ((c ^ sw) << 4)));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  const GroupScale g = make_scale<FMT>(m);
  const uint32_t dst = afp8 + r * 128;
  bool slow = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint2 c0 = quant8_fast<FMT>(ld_shared_v4(src + (((2 * k) ^ sw) << 4)), g, slow);
    const uint2 c1 = quant8_fast<FMT>(ld_shared_v4(src + (((2 * k + 1) ^ sw) << 4)), g, slow);
    st_shared_v4(dst + (((4 * h + k) ^ sw) << 4), c0.x, c0.y, c1.x, c1.y);
  }
  if (FMT == kFmtFp32 && __any_sync(0xffffffffu, slow)) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint2 c0 = quant8_exact<FMT>(ld_shared_v4(src + (((2 * k) ^ sw) << 4)), g);
      const uint2 c1 = quant8_exact<FMT>(ld_shared_v4(src + (((2 * k + 1) ^ sw) << 4)), g);
      st_shared_v4(dst + (((4 * h + k) ^ sw) << 4), c0.x, c0.y, c1.x, c1.y);
    }
  }
  if (h == 0) {
    if constexpr (FMT == kFmtFp32)
      ring_sa[r] = g.s;
    else
      *reinterpret_cast<uint32_t*>(sf_image + 16 * (r & 31) + 4 * (r >> 5)) = g.byte * 0x01010101u;
  }
}

template <int FMT, bool B_KMAJOR, bool B_ROW>
__global__ void __launch_bounds__(kThreads, 1) gemm_pair_fused_kernel(const __grid_constant__ Params p) {
  using namespace fusedk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool kFp32 = (FMT == kFmtFp32);
  constexpr int S = F_STAGES;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + F_kOffBar);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto full_bar = [&](int s) { return bar(s); };
  auto fullsc_bar = [&](int s) { return bar(S + s); };
  auto empty_bar = [&](int s) { return bar(2 * S + s); };
  auto sfmma_bar = [&](int s) { return bar(3 * S + s); };
  auto aready_bar = [&](int s) { return bar(4 * S + s); };
  auto aconv_bar = [&](int q) { return bar(5 * S + q); };
  auto sfready_bar = [&](int q) { return bar(5 * S + kRing + q); };
  auto tfull_bar = [&](int b) { return bar(5 * S + 2 * kRing + b); };
  auto tempty_bar = [&](int b) { return bar(5 * S + 2 * kRing + 2 + b); };
  const uint32_t final_bar = bar(5 * S + 2 * kRing + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + F_kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + F_kOffMisc + 4);
  const WaitGuard guard{abort_flag, p.status, p.limit_ns};
  auto ring = [&](int q) { return smem + F_kOffRing + q * F_kRingBytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(fullsc_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sfmma_bar(s), 2);
      mbar_init(aready_bar(s), 2 * kEpiWarps);
    }
    for (int q = 0; q < kRing; ++q) {
      mbar_init(aconv_bar(q), kEpiWarps);
      mbar_init(sfready_bar(q), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const ClockStamp clk0 = clock_begin(p);
  const uint32_t tmem_base = *tmem_holder;
  const int KB = p.num_kb;
  const int cl = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(nclusters_x());
  constexpr int BMC = 128, TBN = 256, BNC = 128;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tmA);
      prefetch_tensormap(&p.tmB);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cl; ok && tile < p.num_tiles; tile += ncl) {
        int mb, nb;
        tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
        const int32_t row0 = mb * (2 * BMC) + BMC * static_cast<int>(rank);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, guard, kTimeoutProducer)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * F_kTileB);
          const uint32_t fb = mapa_shared(full_bar(s), 0);
          const uint32_t sb = smem_u32(smem + F_kOffB + s * F_kTileB);
          if (B_KMAJOR)
            tma_load_2d_pair(sb, &p.tmB, fb, kb * BK, nb * TBN + BNC * static_cast<int>(rank));
          else
            tma_load_2d_pair(sb, &p.tmB, fb, nb * TBN + BNC * static_cast<int>(rank), kb * BK);
          const uint32_t esz = kFp32 ? 4u : 1u;
          uint32_t b_sc_bytes = 0;
          if (B_ROW) {
            const int64_t left = p.sb_len - static_cast<int64_t>(nb) * TBN;
            b_sc_bytes = static_cast<uint32_t>(left < TBN ? left : TBN) * esz;
          }
          mbar_arrive_expect_tx(fullsc_bar(s), F_kTileAbf + b_sc_bytes);
          const uint32_t sab = smem_u32(smem + F_kOffAbf + s * F_kTileAbf);
          tma_load_2d(sab, &p.tmA, fullsc_bar(s), kb * BK, row0);
          tma_load_2d(sab + F_kTileAbf / 2, &p.tmA, fullsc_bar(s), kb * BK + 64, row0);
          if (B_ROW) {
            uint8_t* slot = smem + F_kOffSlot + s * kSlotBytes;
            const uint8_t* gb = static_cast<const uint8_t*>(p.sB) +
                                (kb * p.sb_stride_k + static_cast<int64_t>(nb) * TBN) * esz;
            bulk_load(smem_u32(slot + kSlotRawB), gb, b_sc_bytes, fullsc_bar(s));
          }
        }
      }
      const uint32_t total = it;
      for (uint32_t j = (total > S ? total - S : 0); j < total; ++j) {
        mbar_wait(empty_bar(j % S), (j / S) & 1, guard, kTimeoutTeardown);
        mbar_wait(fullsc_bar(j % S), (j / S) & 1, guard, kTimeoutTeardown);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // Warp-uniform loop; one elected lane issues (as in the pair kernel).
    if (leader) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t idesc = kFp32 ? idesc_f8(2 * BMC, TBN, !B_KMAJOR) : idesc_mxf8(2 * BMC, TBN, !B_KMAJOR);
      for (int tile = cl; ok && tile < p.num_tiles; tile += ncl, ++tcount) {
        if (!kFp32) {
          if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(0), (tcount & 1) ^ 1, guard, kTimeoutMma))) { ok = false; break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          uint32_t d = tmem_base;
          if (kFp32) {
            const uint32_t b = it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(b), ((it >> 1) & 1) ^ 1, guard, kTimeoutMma))) { ok = false; break; }
            d = tmem_base + b * 256;
          }
          if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
          if (!__all_sync(0xffffffffu, mbar_wait(aready_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
          if (!kFp32 && !__all_sync(0xffffffffu, mbar_wait(sfmma_bar(s), ph, guard, kTimeoutMma))) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + F_kOffA + s * F_kTileA);
          const uint32_t sb = smem_u32(smem + F_kOffB + s * F_kTileB);
          const uint32_t sf_a = tmem_base + kTmemSf + 16 * s;
          const uint32_t sf_b = sf_a + 8;
          if (elect_one()) {
            if (!kFp32) {
              const uint32_t tm = smem_u32(smem + F_kOffSlot + s * kSlotBytes + kSlotTm);
              tc_cp_32x128b_warpx4_pair(sf_a, smem_desc(tm, 0, 128, kLayoutNone));
              tc_cp_32x128b_warpx4_pair(sf_b, smem_desc(tm + 512, 0, 128, kLayoutNone));
              tc_cp_32x128b_warpx4_pair(sf_b + 4, smem_desc(tm + 1024, 0, 128, kLayoutNone));
            }
#pragma unroll
            for (int k4 = 0; k4 < BK / 32; ++k4) {
              const uint64_t adesc = smem_desc(sa + 32 * k4, 16, 1024, kLayoutSw128);
              const uint64_t bdesc = B_KMAJOR ? smem_desc(sb + 32 * k4, 16, 1024, kLayoutSw128)
                                              : smem_desc(sb + 4096 * k4, F_kTileB, 1024, kLayoutSw128);
              if (kFp32)
                mma_f8_pair(d, adesc, bdesc, idesc, k4 > 0 ? 1u : 0u);
              else
                mma_mxf8_pair(d, adesc, bdesc, idesc, sf_a, sf_b, (kb > 0 || k4 > 0) ? 1u : 0u);
            }
            tc_commit_pair(empty_bar(s), 0x3);
            if (kFp32) tc_commit_pair(tfull_bar(it & 1), 0x3);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (!kFp32 && elect_one()) tc_commit_pair(tfull_bar(0), 0x3);
        __syncwarp();
      }
      if (elect_one()) tc_commit_pair(final_bar, 0x1);
      __syncwarp();
      mbar_wait(final_bar, 0, guard, kTimeoutTeardown);
    }
  } else if (warp == 2) {
    // ------------------------------------- B scale staging (A is converted)
    uint32_t it = 0;
    bool ok = true;
    const uint32_t sfmma_leader_base = mapa_shared(sfmma_bar(0), 0);
    for (int tile = cl; ok && tile < p.num_tiles; tile += ncl) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
      uint32_t cur0 = 0, cur1 = 0, nxt0 = 0, nxt1 = 0;
      if (!B_ROW) {
        load_block_scales(p, nb, 0, kFp32, cur0, cur1);
        load_block_scales(p, nb, 32, kFp32, nxt0, nxt1);
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!B_ROW && kb > 0 && (kb & 31) == 0) {
          cur0 = nxt0;
          cur1 = nxt1;
          load_block_scales(p, nb, kb + 32, kFp32, nxt0, nxt1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(fullsc_bar(s), ph, guard, kTimeoutScale))) { ok = false; break; }
        uint8_t* slot = smem + F_kOffSlot + s * kSlotBytes;
        uint32_t b0 = 0, b1 = 0;
        if (!B_ROW) {
          b0 = __shfl_sync(0xffffffffu, cur0, kb & 31);
          b1 = __shfl_sync(0xffffffffu, cur1, kb & 31);
        }
        if (kFp32) {
          const int q = it % kRing;
          if (!B_ROW && lane == 0) {
            reinterpret_cast<uint32_t*>(ring(q) + 512)[0] = b0;
            reinterpret_cast<uint32_t*>(ring(q) + 512)[1] = b1;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(sfready_bar(q));
        } else {
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
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(sfmma_leader_base + 8 * s);
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------- A quantization + epilogue warps
    const int ew = warp - kEpiWarp0;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int row_in_tile = 32 * quarter + lane;
    const int e = ew * 32 + lane;  // converter thread: row e / 2, column half e % 2
    uint8_t* stage = smem + F_kOffStage + ew * kStageBytes;
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    const uint32_t aready_leader0 = mapa_shared(aready_bar(0), 0);
    uint32_t it = 0, tcount = 0;
    bool ok = true;

    // Quantize the BF16 A tile of iteration `ci` (stage ci % S).
    auto convert = [&](uint32_t ci) -> bool {
      const int s = ci % S;
      if (!__all_sync(0xffffffffu, mbar_wait(fullsc_bar(s), (ci / S) & 1, guard, kTimeoutEpilogue))) return false;
      float* ring_sa = reinterpret_cast<float*>(ring(ci % kRing));
      uint8_t* sf_image = smem + F_kOffSlot + s * kSlotBytes + kSlotTm;
      fused_convert_half<FMT>(smem_u32(smem + F_kOffAbf + s * F_kTileAbf), smem_u32(smem + F_kOffA + s * F_kTileA),
                              e >> 1, e & 1, ring_sa, sf_image);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(aready_leader0 + 8 * s);
        if (kFp32) mbar_arrive(aconv_bar(ci % kRing));
      }
      return true;
    };

    for (int tile = cl; ok && tile < p.num_tiles; tile += ncl, ++tcount) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, p.group_m, mb, nb);
      float2 acc[64];
      const uint32_t it0 = it;
      if (kFp32) {
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int j = 0; j <= KB; ++j) {
          if (j < KB && !convert(it0 + j)) { ok = false; break; }
          if (j == 0) continue;
          const uint32_t pi = it0 + j - 1;  // promote K block j - 1
          const uint32_t b = pi & 1;
          const int q = pi % kRing;
          if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(b), (pi >> 1) & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
          if (!__all_sync(0xffffffffu, mbar_wait(aconv_bar(q), (pi / kRing) & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
          if (!__all_sync(0xffffffffu, mbar_wait(sfready_bar(q), (pi / kRing) & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
          tc_fence_after();
          const float sa = reinterpret_cast<const float*>(ring(q))[row_in_tile];
          const uint8_t* slot = smem + F_kOffSlot + (pi % S) * kSlotBytes;
          const uint32_t cbase = tmem_base + lane_addr + b * 256 + half * 128;
          const float2 sa2 = make_float2(sa, sa);
          float2 f2 = sa2;
          if (!B_ROW) {
            const float f = sa * reinterpret_cast<const float*>(ring(q) + 512)[half];
            f2 = make_float2(f, f);
          }
          if (!B_ROW) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float r[32];
              tmem_ld_32x32b_x32f(cbase + 32 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                acc[16 * c + i] = __ffma2_rn(make_float2(r[2 * i], r[2 * i + 1]), f2, acc[16 * c + i]);
            }
          } else {
            // per-column B scales: 16-column loads keep the staging small
            // enough for the 128 accumulators to stay in registers
            const float2* sbv = reinterpret_cast<const float2*>(slot + kSlotRawB) + half * 64;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float r[16];
              tmem_ld_32x32b_x16f(cbase + 16 * c, r);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i)
                acc[8 * c + i] = __ffma2_rn(make_float2(r[2 * i], r[2 * i + 1]), __fmul2_rn(sa2, sbv[8 * c + i]),
                                            acc[8 * c + i]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * b);
        }
        if (!ok) break;
        it = it0 + KB;
      } else {
        for (int j = 0; j < KB; ++j)
          if (!convert(it0 + j)) { ok = false; break; }
        if (!ok) break;
        it = it0 + KB;
        if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(0), tcount & 1, guard, kTimeoutEpilogue))) { ok = false; break; }
        tc_fence_after();
        const uint32_t cbase = tmem_base + lane_addr + half * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32f(cbase + 32 * c, &acc[16 * c].x);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader0);
      }
      const int m0 = mb * (2 * BMC) + BMC * static_cast<int>(rank) + 32 * quarter;
      store_tile(p, acc, stage, lane, m0, nb * TBN + half * 128);
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  clock_end(p, clk0);
}

// ------------------------------------------------------------------- host --
__device__ int g_device_status;

struct DeviceInfo {
  unsigned long long ctx = 0;  // context the cached addresses and attributes belong to
  unsigned long long* clk = nullptr;  // clock counters of later launches (fp8bq_set_clock_counters)
  int sms = 0;
  int64_t l2_bytes = 0;
  int* status = nullptr;
  bool attr_set[8] = {};
  bool pair_attr_set[12] = {};
  int pair_clusters[12] = {};
  bool fused_attr_set[8] = {};
  int fused_clusters[8] = {};
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
  // The status word's address and the kernels' attributes belong to one
  // context: a new context on this device (after cudaDeviceReset, say) is
  // set up again.
  const unsigned long long id = current_context_id();
  if (d.sms == 0 || id == 0 || d.ctx != id) {
    d = DeviceInfo{};
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
      d.sms = 0;
      return e;
    }
    int l2 = 0;
    e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    if (e != cudaSuccess) {
      d.sms = 0;
      return e;
    }
    d.l2_bytes = l2;
    void* sym = nullptr;
    e = cudaGetSymbolAddress(&sym, g_device_status);  // makes the device's context current if none is
    if (e != cudaSuccess) {
      d.sms = 0;
      return e;
    }
    d.status = static_cast<int*>(sym);
    d.ctx = current_context_id();
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

// Whole tiles take ceil(T / C) rounds on C clusters, the last one R / C full
// (R = T mod C).  With a workspace, the R tiles of that round are split along
// K over all C clusters (about W + R / C rounds, W = T / C) when there is at
// least one full round, the split saves more than 5% of the launch, each
// cluster gets at least four K blocks and the workspace has a slot per
// cluster.  Not for FP32 accumulation.  (With fewer tiles than clusters,
// measured on the layer's O-projection weight gradient, every tile splits
// into two pieces and the launch got slower, not faster: the SM clock the
// tensor cores sustain drops as more of them run, which takes back most of
// what the idle clusters would have added.)
bool split_tiles(Params& prm, int C, const GemmProblem& pr) {
  const int T = prm.num_tiles, W = T / C, R = T % C;
  const int64_t slots = pr.ws != nullptr ? pr.ws_bytes / kWsSlotBytes : 0;
  if (pr.acc_f32 || W == 0 || R == 0 || slots < C) return false;
  if (20LL * (C - R) <= static_cast<int64_t>(C) * (W + 1)) return false;
  if (static_cast<int64_t>(R) * prm.num_kb < 4LL * C) return false;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {256, static_cast<cuuint64_t>(slots) * 256};
  cuuint64_t strides[1] = {256 * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  if (fn(&prm.tmW, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, pr.ws, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  prm.ws = static_cast<float*>(pr.ws);
  prm.ws_flag = reinterpret_cast<int*>(static_cast<uint8_t*>(pr.ws) + slots * kWsTileBytes);
  prm.dp_tiles = W * C;
  return true;
}

template <int FMT, bool BK_, bool BR_, bool ACC_ = false>
cudaError_t launch_pair_variant(Params& prm, const GemmProblem& pr, DeviceInfo* di, int slot, cudaStream_t stream) {
  auto kern = gemm_pair_kernel<FMT, BK_, BR_, ACC_>;
  constexpr uint32_t kSmem = pairk::Cfg<FMT, ACC_>::kSmemAlloc;
  if (!di->pair_attr_set[slot]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t occ = {};
    occ.gridDim = dim3(2 * 148, 1, 1);
    occ.blockDim = dim3(pairk::Cfg<FMT, ACC_>::kThreads, 1, 1);
    occ.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    occ.attrs = attr;
    occ.numAttrs = 1;
    int ncl = 0;
    e = cudaOccupancyMaxActiveClusters(&ncl, kern, &occ);
    if (e != cudaSuccess) return e;
    if (ncl <= 0) return cudaErrorInvalidConfiguration;
    di->pair_clusters[slot] = ncl;
    di->pair_attr_set[slot] = true;
  }
  int ncl = prm.num_tiles < di->pair_clusters[slot] ? prm.num_tiles : di->pair_clusters[slot];
  if (split_tiles(prm, di->pair_clusters[slot], pr)) ncl = di->pair_clusters[slot];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl, 1, 1);
  cfg.blockDim = dim3(pairk::Cfg<FMT, ACC_>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int FMT, bool BK_, bool BR_>
cudaError_t launch_fused_variant(const Params& prm, DeviceInfo* di, int slot, cudaStream_t stream) {
  auto kern = gemm_pair_fused_kernel<FMT, BK_, BR_>;
  if (!di->fused_attr_set[slot]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, fusedk::F_kSmemAlloc);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t occ = {};
    occ.gridDim = dim3(2 * 148, 1, 1);
    occ.blockDim = dim3(kThreads, 1, 1);
    occ.dynamicSmemBytes = fusedk::F_kSmemAlloc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    occ.attrs = attr;
    occ.numAttrs = 1;
    int ncl = 0;
    e = cudaOccupancyMaxActiveClusters(&ncl, kern, &occ);
    if (e != cudaSuccess) return e;
    if (ncl <= 0) return cudaErrorInvalidConfiguration;
    di->fused_clusters[slot] = ncl;
    di->fused_attr_set[slot] = true;
  }
  const int ncl = prm.num_tiles < di->fused_clusters[slot] ? prm.num_tiles : di->fused_clusters[slot];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = fusedk::F_kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
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
  if (!pr.a.k_major || !pr.a.row_groups || (pr.b.row_groups && !pr.b.k_major)) {
    *unsupported = true;
    return cudaSuccess;
  }
  DeviceInfo* di = nullptr;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;

  // M <= 128 runs the single-CTA kernel (128 x 256 tiles); larger M, and any
  // BF16 A (fused quantize-on-load), runs CTA pairs (256 x 256 tiles, 128 rows
  // of A and of B per CTA).
  const bool fused = pr.a.bf16;
  const bool mx = pr.a.mx;  // 1x32 blocks on both operands (checked at the ABI)
  if (mx && (fused || !pr.b.mx || !pr.b.k_major || !pr.b.row_groups)) {
    *unsupported = true;
    return cudaSuccess;
  }
  // FP32 accumulation (D += A B^T) is built for the weight-gradient layout:
  // both operands row groups, K-major, on CTA pairs
  const bool acc = pr.acc_f32;
  if (acc && (fused || !pr.a.row_groups || !pr.b.row_groups || !pr.b.k_major)) {
    *unsupported = true;
    return cudaSuccess;
  }
  // a mixed pair (one operand's scales UE8M0, the other's FP32) decodes the
  // UE8M0 bytes in the CTA-pair kernel's scale staging
  const bool mixed = pr.a_u8 || pr.b_u8;
  if (mixed && (fused || mx || pr.fmt != kFmtFp32)) {
    *unsupported = true;
    return cudaSuccess;
  }
  const bool pair = fused || mx || acc || mixed || pr.M > 128;
  Params prm;
  memset(&prm, 0, sizeof(prm));
  if (fused) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(pr.K), static_cast<cuuint64_t>(pr.M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(pr.a.ld) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(&prm.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pr.a.data), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  } else if (!encode_2d(&prm.tmA, pr.a.data, pr.K, pr.M, pr.a.ld, BK, BM)) {
    return cudaErrorInvalidValue;
  }
  if (pr.b.k_major) {
    if (!encode_2d(&prm.tmB, pr.b.data, pr.K, pr.N, pr.b.ld, BK, pair ? pairk::P_BNC : BN))
      return cudaErrorInvalidValue;
  } else {
    if (!encode_2d(&prm.tmB, pr.b.data, pr.N, pr.K, pr.b.ld, 128, BK)) return cudaErrorInvalidValue;
  }
  {
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    // BF16 D: 64 x 32 boxes; FP32 D (accumulating): 32 x 32 boxes; both 128-byte rows
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(pr.N), static_cast<cuuint64_t>(pr.M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(pr.ldd) * (acc ? 4 : 2)};
    cuuint32_t box[2] = {acc ? 32u : 64u, 32};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(&prm.tmD, acc ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pr.d,
                    dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  prm.sA = pr.a.scales;
  prm.sB = pr.b.scales;
  prm.sa_stride_k = pr.a.s_stride_k;
  prm.sb_stride_k = pr.b.s_stride_k;
  prm.sb_stride_r = pr.b.s_stride_r;
  prm.sb_len = pr.b.row_groups ? pr.b.s_stride_k : 0;
  if (!mx && pair && !fused && pr.fmt == kFmtUe8m0) {
    // UE8M0 scales of the CTA-pair kernel travel in groups of four K blocks:
    // byte matrices [K/128][ld], boxes of 128 (A) or 256 (row-group B) rows
    // by 4 K blocks; past-the-end rows and K blocks read as zeros
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const void* sp[2] = {pr.a.scales, pr.b.scales};
    const int64_t ld[2] = {pr.a.s_stride_k, pr.b.s_stride_k};
    const uint32_t boxc[2] = {128, 256};
    CUtensorMap* maps[2] = {&prm.tmSA, &prm.tmSB};
    for (int i = 0; i < (pr.b.row_groups ? 2 : 1); ++i) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(ld[i]), static_cast<cuuint64_t>(pr.K / 128)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld[i])};
      cuuint32_t box[2] = {boxc[i], 4};
      cuuint32_t es[2] = {1, 1};
      CUresult r = fn(maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(sp[i]), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
  }
  if (mx) {
    // 1x32 scale arrays as byte matrices [K/32][ld]; boxes of 4 scale rows
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const void* sp[2] = {pr.a.scales, pr.b.scales};
    const int64_t ld[2] = {pr.a.s_stride_k, pr.b.s_stride_k};
    const uint32_t boxc[2] = {128, 256};
    CUtensorMap* maps[2] = {&prm.tmSA, &prm.tmSB};
    for (int i = 0; i < 2; ++i) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(ld[i]), static_cast<cuuint64_t>(pr.K / 32)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld[i])};
      cuuint32_t box[2] = {boxc[i], 4};
      cuuint32_t es[2] = {1, 1};
      CUresult r = fn(maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(sp[i]), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
  }
  prm.nb_blocks = (pr.N + 127) / 128;
  prm.D = static_cast<uint16_t*>(pr.d);
  prm.ldd = pr.ldd;
  prm.M = static_cast<int>(pr.M);
  prm.N = static_cast<int>(pr.N);
  prm.K = static_cast<int>(pr.K);
  const int64_t tile_m = pair ? 2 * pairk::P_BMC : BM;
  prm.num_m = static_cast<int>((pr.M + tile_m - 1) / tile_m);
  prm.num_n = static_cast<int>((pr.N + BN - 1) / BN);
  prm.num_tiles = prm.num_m * prm.num_n;
  prm.num_kb = static_cast<int>(pr.K / BK);
  prm.dp_tiles = prm.num_tiles;  // nothing split unless the pair launcher splits
  prm.status = di->status;
  prm.limit_ns = pr.wait_limit_ns != 0 ? pr.wait_limit_ns : 2000000000ull;  // 2 s per wait
  prm.a_u8 = pr.a_u8 ? 1 : 0;
  prm.b_u8 = pr.b_u8 ? 1 : 0;
  prm.withhold_cluster = pr.withhold_cluster;
  {
    // L2 priorities: the output (written once) goes first, and so does A
    // when it is larger than the L2 (streamed: each of its row blocks read
    // by the tiles of one wave; the gate/up data and weight gradients, A =
    // dY at 201 MB, run 1-1.5% faster).  A smaller A keeps the normal
    // priority (marked first, the down projection's forward, A = 100 MB,
    // ran 3% slower), and so does B even when large: its tiles are read by
    // every M block of a raster group, and marked first they lost that reuse
    // to the output stream (LM head forward, B = the 311 MB weight: 4.97 ms
    // against 4.46 ms unmarked).
    const int64_t half_l2 = di->l2_bytes / 2;
    const int64_t a_bytes = pr.M * pr.K * (pr.a.bf16 ? 2 : 1);
    uint32_t h = kHintDFirst;
    if (a_bytes > di->l2_bytes) h |= kHintAFirst;
    // raster: groups of kGroupM M blocks share each B tile among them; when all of
    // A fits in half the L2 and B does not (the LM head: 33.5 MB of
    // activations against a 311 MB weight), one group spans every M block,
    // so that each B tile is read from HBM once while A stays in L2
    const int64_t b_bytes = pr.N * pr.K;
    prm.group_m = (di->l2_bytes > 0 && a_bytes <= half_l2 && b_bytes > half_l2) ? prm.num_m : kGroupM;
    prm.l2_hints = di->l2_bytes > 0 ? h : 0;
  }
  prm.clk = di->clk;
  const int grid = prm.num_tiles < di->sms ? prm.num_tiles : di->sms;

  const bool fp32 = pr.fmt == kFmtFp32;
  const bool bk = pr.b.k_major;
  const bool br = pr.b.row_groups;
  if (fused) {
    if (fp32) {
      if (bk && !br) return launch_fused_variant<kFmtFp32, true, false>(prm, di, 0, stream);
      if (!bk && !br) return launch_fused_variant<kFmtFp32, false, false>(prm, di, 1, stream);
      return launch_fused_variant<kFmtFp32, true, true>(prm, di, 2, stream);
    }
    if (bk && !br) return launch_fused_variant<kFmtUe8m0, true, false>(prm, di, 3, stream);
    if (!bk && !br) return launch_fused_variant<kFmtUe8m0, false, false>(prm, di, 4, stream);
    return launch_fused_variant<kFmtUe8m0, true, true>(prm, di, 5, stream);
  }
  if (acc) {
    if (mx) return launch_pair_variant<kFmtMx, true, true, true>(prm, pr, di, 9, stream);
    if (fp32) return launch_pair_variant<kFmtFp32, true, true, true>(prm, pr, di, 7, stream);
    return launch_pair_variant<kFmtUe8m0, true, true, true>(prm, pr, di, 8, stream);
  }
  if (mx) return launch_pair_variant<kFmtMx, true, true>(prm, pr, di, 6, stream);
  if (pair) {
    if (fp32) {
      if (bk && !br) return launch_pair_variant<kFmtFp32, true, false>(prm, pr, di, 0, stream);
      if (!bk && !br) return launch_pair_variant<kFmtFp32, false, false>(prm, pr, di, 1, stream);
      return launch_pair_variant<kFmtFp32, true, true>(prm, pr, di, 2, stream);
    }
    if (bk && !br) return launch_pair_variant<kFmtUe8m0, true, false>(prm, pr, di, 3, stream);
    if (!bk && !br) return launch_pair_variant<kFmtUe8m0, false, false>(prm, pr, di, 4, stream);
    return launch_pair_variant<kFmtUe8m0, true, true>(prm, pr, di, 5, stream);
  }
  if (fp32) {
    if (bk && !br) return launch_variant<kFmtFp32, true, false>(prm, grid, di, 0, stream);
    if (!bk && !br) return launch_variant<kFmtFp32, false, false>(prm, grid, di, 1, stream);
    return launch_variant<kFmtFp32, true, true>(prm, grid, di, 2, stream);
  }
  if (bk && !br) return launch_variant<kFmtUe8m0, true, false>(prm, grid, di, 3, stream);
  if (!bk && !br) return launch_variant<kFmtUe8m0, false, false>(prm, grid, di, 4, stream);
  return launch_variant<kFmtUe8m0, true, true>(prm, grid, di, 5, stream);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return encode_fn(); }

cudaError_t device_sm_count(int* sms) {
  DeviceInfo* di = nullptr;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  *sms = di->sms;
  return cudaSuccess;
}

cudaError_t set_clock_counters(unsigned long long* counters) {
  DeviceInfo* di = nullptr;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_mu);
  di->clk = counters;
  return cudaSuccess;
}

cudaError_t device_status_word(int** status) {
  DeviceInfo* di = nullptr;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  *status = di->status;
  return cudaSuccess;
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
