// internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "fp8bq.h"

namespace fp8bq {

// FP8BQ_OK for cudaSuccess; otherwise records `e` as this thread's last CUDA
// error (what fp8bq_last_cuda_error() returns) and gives FP8BQ_ERR_CUDA.
// Every entry point maps its CUDA failures through this one function.
int cuda_status(cudaError_t e);

// Unique identifier of the CUDA context current on the calling thread
// (cuCtxGetId: never reused within the process, unlike the context handle),
// or 0 when no context is current or the driver entry point is missing.
// Device addresses of the library's __device__ objects and per-function
// attributes belong to one context; caches of them are keyed on this.
unsigned long long current_context_id();

inline int64_t round_up128(int64_t r) { return (r + 127) / 128 * 128; }

// TMA-fed activation quantizer: row-group codes (q != nullptr), token-group
// codes (qt != nullptr), or both from one read of X; groups of `group` = 128
// or (UE8M0 only) 32 values.
cudaError_t launch_quant_tiles(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* s_rows,
                               void* qt, void* s_cols, int fmt, int group, cudaStream_t stream);

// One job of a grouped quantization launch: an activation X [rows, cols]
// quantized in row groups (q), token groups (qt) or both, or (block) a weight
// W [rows, cols] in 128x128 blocks (q, s_rows = scales [cols/128][ceil(rows/128)]).
struct QuantJob {
  const void* x;
  int64_t rows, cols, ldx;
  void* q;
  void* s_rows;
  void* qt;
  void* s_cols;
  bool block;
};
// Up to 8 jobs in one persistent launch (one format, groups of 128).
cudaError_t launch_quant_group(const QuantJob* jobs, int njobs, int fmt, cudaStream_t stream);

// SwiGLU of [gate | up] fused with the quantization of its output h
// (row groups, and token groups when qt != nullptr); h optionally stored;
// exact: h rounded once from its exact value.
cudaError_t launch_swiglu_quant(const void* gu, int64_t M, int64_t F, int64_t ldgu, void* h, void* q, void* s_rows,
                                void* qt, void* s_cols, int fmt, bool exact, cudaStream_t stream);
cudaError_t launch_rmsnorm_quant(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
                                 float* rstd, void* h, void* q, void* s_rows, void* qt, void* s_cols, int fmt,
                                 cudaStream_t stream);
// The same with h rounded once from its exact value; rstd64 [M] in float64.
cudaError_t launch_rmsnorm_quant_exact(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                       double eps, double* rstd64, void* h, void* q, void* s_rows, void* qt,
                                       void* s_cols, int fmt, cudaStream_t stream);

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
  // Kernel family: kFmtUe8m0 (both operands UE8M0: block-scaled MMA) or
  // kFmtFp32 (promotion path: at least one operand has FP32 scales; an
  // operand with UE8M0 scales then has them decoded to 2^e, a_u8 / b_u8).
  int fmt;
  bool a_u8 = false, b_u8 = false;
  bool acc_f32;   // D is FP32 and accumulated into (D += A B^T); else BF16 D = A B^T
  void* ws = nullptr;    // split-tile workspace (flags zero between calls), or none
  int64_t ws_bytes = 0;
  // Test hooks, off in every product call: the split-tile piece of this CTA
  // pair stores its partial sum but never raises its flags (-1: none), and
  // the bounded waits' limit in ns (0: the default 2 s).
  int withhold_cluster = -1;
  uint64_t wait_limit_ns = 0;
};

// Checks the arguments of fp8bq_gemm_ws (all but the workspace) and the
// device, and fills `p`; returns FP8BQ_OK or the call's error status.
int validate_gemm(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N, int64_t K,
                  int64_t ldd, uint32_t flags, GemmProblem* p);
// Launches a validated problem; returns a status.
int run_gemm(const GemmProblem& p, cudaStream_t stream);

// Split-tile workspace: one slot of a 256 x 256 FP32 partial sum per CTA
// pair, then 16 int flags per slot (one per epilogue warp slice of the pair).
constexpr int64_t kWsTileBytes = 256 * 256 * 4;
constexpr int64_t kWsSlotBytes = kWsTileBytes + 16 * 4;

// Launches the GEMM; returns a cudaError_t (cudaSuccess on success).  Sets
// *unsupported when the operand combination is not built.
cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream, bool* unsupported);

// GEMM launches on the current device (in its current context) issued after
// this call add their CTAs' SM cycles and nanoseconds to counters[0..1]
// (nullptr: stop).
cudaError_t set_clock_counters(unsigned long long* counters);

// Device status word of the GEMM kernels (0 = ok, else a timeout code).
// Reads and clears it after synchronizing `stream`.
cudaError_t read_and_clear_device_status(cudaStream_t stream, int* status);

}  // namespace fp8bq
