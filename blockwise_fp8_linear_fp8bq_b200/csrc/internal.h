// internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

namespace fp8bq {

inline int64_t round_up128(int64_t r) { return (r + 127) / 128 * 128; }

cudaError_t launch_quant_weight(const void* w, int64_t N, int64_t K, int64_t ldw, void* q,
                                void* scales, int fmt, cudaStream_t stream);
// TMA-fed activation quantizer: row-group codes (q != nullptr), token-group
// codes (qt != nullptr), or both from one read of X; groups of `group` = 128
// or (UE8M0 only) 32 values.
cudaError_t launch_quant_tiles(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* s_rows,
                               void* qt, void* s_cols, int fmt, int group, cudaStream_t stream);

// SwiGLU of [gate | up] fused with the quantization of its output h
// (row groups, and token groups when qt != nullptr); h optionally stored.
cudaError_t launch_swiglu_quant(const void* gu, int64_t M, int64_t F, int64_t ldgu, void* h, void* q, void* s_rows,
                                void* qt, void* s_cols, int fmt, cudaStream_t stream);
cudaError_t launch_rmsnorm_quant(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
                                 float* rstd, void* h, void* q, void* s_rows, void* qt, void* s_cols, int fmt,
                                 cudaStream_t stream);

// Driver entry point of cuTensorMapEncodeTiled (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
// Multiprocessor count of the current device (cached).
cudaError_t device_sm_count(int* sms);
// Device address of the kernels' status word on the current device.
cudaError_t device_status_word(int** status);

// A validated GEMM problem, in the library's internal form.
struct GemmOperand {
  const void* data;
  int64_t ld;
  bool bf16;     // operand A given as BF16 (quantized inside the GEMM)
  bool k_major;  // contraction contiguous
  const void* scales;
  bool row_groups;  // 1x128 (or, with mx, 1x32) row groups, else 128x128 blocks
  bool mx;          // 1x32 row groups (MX blocks, UE8M0)
  int64_t s_stride_k;
  int64_t s_stride_r;
};

struct GemmProblem {
  GemmOperand a, b;
  void* d;
  int64_t M, N, K, ldd;
  int fmt;        // kFmtFp32 / kFmtUe8m0 (both operands)
  bool acc_f32;   // D is FP32 and accumulated into (D += A B^T); else BF16 D = A B^T
  void* ws = nullptr;    // split-tile workspace (flags zero between calls), or none
  int64_t ws_bytes = 0;
};

// Split-tile workspace: one slot of a 256 x 256 FP32 partial sum per CTA
// pair, then 16 int flags per slot (one per epilogue warp slice of the pair).
constexpr int64_t kWsTileBytes = 256 * 256 * 4;
constexpr int64_t kWsSlotBytes = kWsTileBytes + 16 * 4;

// Launches the GEMM; returns a cudaError_t (cudaSuccess on success).  Sets
// *unsupported when the operand combination is not built.
cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream, bool* unsupported);

// Device status word of the GEMM kernels (0 = ok, else a timeout code).
// Reads and clears it after synchronizing `stream`.
cudaError_t read_and_clear_device_status(cudaStream_t stream, int* status);

}  // namespace fp8bq
