// fp8bq_api.cu -- the C ABI declared in include/fp8bq.h: argument checks,
// status codes and dispatch to the kernels.  Nothing here allocates device
// memory or synchronizes, except fp8bq_check().
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fp8bq.h"
#include "fp8bq_testing.h"
#include "internal.h"
#include "quant_math.cuh"

namespace {
thread_local int t_last_cuda_error = 0;
}  // namespace

namespace fp8bq {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FP8BQ_OK;
  t_last_cuda_error = static_cast<int>(e);
  return FP8BQ_ERR_CUDA;
}

unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace fp8bq

namespace {

using fp8bq::cuda_status;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_fmt(int fmt) { return fmt == FP8BQ_SCALE_FP32 || fmt == FP8BQ_SCALE_UE8M0; }

// Kernels need an sm_100 device; checked once per device.
int device_ok() {
  static int cached[64] = {};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= 64) return FP8BQ_ERR_UNSUPPORTED;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_status(e);
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1 ? FP8BQ_OK : FP8BQ_ERR_UNSUPPORTED;
}

int check_quant_args(const void* x, int64_t rows, int64_t cols, int64_t ld, const void* q,
                     const void* scales, int fmt) {
  if (!x || !q || !scales) return FP8BQ_ERR_INVALID_ARG;
  if (!valid_fmt(fmt)) return FP8BQ_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols) return FP8BQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales) || (ld % 8) != 0) return FP8BQ_ERR_ALIGN;
  return FP8BQ_OK;
}

// Operand checks shared by A and B; fills the internal form.
int convert_operand(const fp8bq_operand* op, int64_t rows, int64_t K, bool is_a, fp8bq::GemmOperand* out) {
  if (!op || !op->data) return FP8BQ_ERR_INVALID_ARG;
  if (op->dtype != FP8BQ_E4M3 && op->dtype != FP8BQ_BF16) return FP8BQ_ERR_INVALID_ARG;
  if (op->gran != FP8BQ_GRAN_ROW_1x128 && op->gran != FP8BQ_GRAN_BLOCK_128x128 &&
      op->gran != FP8BQ_GRAN_ROW_1x32)
    return FP8BQ_ERR_INVALID_ARG;
  if (!valid_fmt(op->fmt)) return FP8BQ_ERR_INVALID_ARG;
  const int fmt = op->fmt;
  if (op->k_major != 0 && op->k_major != 1) return FP8BQ_ERR_INVALID_ARG;
  const bool bf16 = op->dtype == FP8BQ_BF16;
  if (bf16 && (!is_a || !op->k_major)) return FP8BQ_ERR_UNSUPPORTED;
  const int64_t esz = bf16 ? 2 : 1;
  if (!aligned16(op->data) || (op->ld * esz) % 16 != 0) return FP8BQ_ERR_ALIGN;
  const int64_t inner = op->k_major ? K : rows;
  if (op->ld < inner) return FP8BQ_ERR_SHAPE;
  if (!bf16) {
    if (!op->scales) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(op->scales)) return FP8BQ_ERR_ALIGN;
    if (op->gran == FP8BQ_GRAN_ROW_1x32 && fmt != FP8BQ_SCALE_UE8M0) return FP8BQ_ERR_UNSUPPORTED;
    if (op->gran == FP8BQ_GRAN_ROW_1x128 || op->gran == FP8BQ_GRAN_ROW_1x32) {
      if (!op->k_major) return FP8BQ_ERR_UNSUPPORTED;
      if (op->s_stride_r != 1 || op->s_stride_k % 128 != 0 || op->s_stride_k < rows)
        return FP8BQ_ERR_SHAPE;
    } else {
      if (is_a) return FP8BQ_ERR_UNSUPPORTED;
      const int64_t nrb = (rows + 127) / 128;
      const int64_t nkb = K / 128;
      const bool plain = op->s_stride_r == 1 && op->s_stride_k >= nrb;
      const bool transposed = op->s_stride_k == 1 && op->s_stride_r >= nkb;
      if (!plain && !transposed) return FP8BQ_ERR_SHAPE;
    }
  } else if (op->gran != FP8BQ_GRAN_ROW_1x128) {
    return FP8BQ_ERR_UNSUPPORTED;  // BF16 A is quantized in 1x128 row groups
  }
  out->data = op->data;
  out->ld = op->ld;
  out->bf16 = bf16;
  out->k_major = op->k_major != 0;
  out->scales = op->scales;
  out->row_groups = op->gran == FP8BQ_GRAN_ROW_1x128 || op->gran == FP8BQ_GRAN_ROW_1x32;
  out->mx = op->gran == FP8BQ_GRAN_ROW_1x32;
  out->s_stride_k = op->s_stride_k;
  out->s_stride_r = op->s_stride_r;
  return FP8BQ_OK;
}

}  // namespace

namespace fp8bq {

int validate_gemm(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N, int64_t K,
                  int64_t ldd, uint32_t flags, GemmProblem* p) {
  if (!A || !B || !D || !p) return FP8BQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(FP8BQ_GEMM_ACCUMULATE_F32)) != 0) return FP8BQ_ERR_INVALID_ARG;
  const bool acc = (flags & FP8BQ_GEMM_ACCUMULATE_F32) != 0;
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0 || ldd < N) return FP8BQ_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return FP8BQ_ERR_SHAPE;
  if (!aligned16(D) || ldd % 8 != 0) return FP8BQ_ERR_ALIGN;
  int st = convert_operand(A, M, K, true, &p->a);
  if (st != FP8BQ_OK) return st;
  st = convert_operand(B, N, K, false, &p->b);
  if (st != FP8BQ_OK) return st;
  if (p->a.mx != p->b.mx) return FP8BQ_ERR_UNSUPPORTED;  // MX blocks on both operands or neither
  // A BF16 A is quantized inside the GEMM in its own format; B must share it
  if (p->a.bf16 && A->fmt != B->fmt) return FP8BQ_ERR_UNSUPPORTED;
  // FP32 accumulation is built for the weight-gradient layout only
  if (acc && (p->a.bf16 || !p->a.row_groups || !p->b.row_groups || !p->b.k_major)) return FP8BQ_ERR_UNSUPPORTED;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  p->d = D;
  p->M = M;
  p->N = N;
  p->K = K;
  p->ldd = ldd;
  // both UE8M0: the block-scaled MMA; otherwise the FP32 promotion path, with
  // an operand's UE8M0 scales decoded to 2^e where they are staged
  const bool both_u8 = A->fmt == FP8BQ_SCALE_UE8M0 && B->fmt == FP8BQ_SCALE_UE8M0;
  p->fmt = both_u8 ? kFmtUe8m0 : kFmtFp32;
  p->a_u8 = !both_u8 && A->fmt == FP8BQ_SCALE_UE8M0;
  p->b_u8 = !both_u8 && B->fmt == FP8BQ_SCALE_UE8M0;
  p->acc_f32 = acc;
  p->ws = nullptr;
  p->ws_bytes = 0;
  return FP8BQ_OK;
}

int run_gemm(const GemmProblem& p, cudaStream_t stream) {
  bool unsupported = false;
  cudaError_t e = launch_gemm(p, stream, &unsupported);
  if (unsupported) return FP8BQ_ERR_UNSUPPORTED;
  return cuda_status(e);
}

}  // namespace fp8bq

extern "C" {

int fp8bq_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                       int fmt, fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, q, scales, nullptr, nullptr, fmt, 128,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_act_t(const void* x, int64_t M, int64_t K, int64_t ldx, void* qt, void* scales,
                         int fmt, fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, qt, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (M % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (K % 8 != 0) return FP8BQ_ERR_ALIGN;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, nullptr, nullptr, qt, scales, fmt, 128,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_act_dual(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                            void* qt, void* scales_t, int fmt, fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  st = check_quant_args(x, M, K, ldx, qt, scales_t, fmt);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0 || M % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, q, scales, qt, scales_t, fmt, 128,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_act_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                          fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, FP8BQ_SCALE_UE8M0);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, q, scales, nullptr, nullptr, FP8BQ_SCALE_UE8M0, 32,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_act_t_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* qt, void* scales,
                            fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, qt, scales, FP8BQ_SCALE_UE8M0);
  if (st != FP8BQ_OK) return st;
  if (M % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (K % 8 != 0) return FP8BQ_ERR_ALIGN;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, nullptr, nullptr, qt, scales, FP8BQ_SCALE_UE8M0, 32,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_act_dual_mx(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, void* scales,
                               void* qt, void* scales_t, fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, FP8BQ_SCALE_UE8M0);
  if (st != FP8BQ_OK) return st;
  st = check_quant_args(x, M, K, ldx, qt, scales_t, FP8BQ_SCALE_UE8M0);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0 || M % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_tiles(x, M, K, ldx, q, scales, qt, scales_t, FP8BQ_SCALE_UE8M0, 32,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_swiglu_quantize(const void* gu, int64_t M, int64_t F, int64_t ldgu, void* h, void* q, void* scales,
                          void* qt, void* scales_t, int fmt, fp8bq_stream_t stream) {
  const bool exact = (fmt & FP8BQ_SWIGLU_EXACT) != 0;
  fmt &= ~FP8BQ_SWIGLU_EXACT;
  int st = check_quant_args(gu, M, 2 * F, ldgu, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if ((qt == nullptr) != (scales_t == nullptr)) return FP8BQ_ERR_INVALID_ARG;
  if (qt != nullptr && (!aligned16(qt) || !aligned16(scales_t))) return FP8BQ_ERR_ALIGN;
  if (h != nullptr && !aligned16(h)) return FP8BQ_ERR_ALIGN;
  if (F % 128 != 0 || (qt != nullptr && M % 128 != 0)) return FP8BQ_ERR_SHAPE;
  if (M == 0 || F == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_swiglu_quant(gu, M, F, ldgu, h, q, scales, qt, scales_t, fmt, exact,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_rmsnorm_quantize(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, float eps,
                           float* rstd, void* h, void* q, void* scales, void* qt, void* scales_t, int fmt,
                           fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (gamma == nullptr || rstd == nullptr) return FP8BQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8BQ_ERR_INVALID_ARG;  // finite, not negative
  if ((qt == nullptr) != (scales_t == nullptr)) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned16(gamma) || (reinterpret_cast<uintptr_t>(rstd) & 3u) != 0) return FP8BQ_ERR_ALIGN;
  if (qt != nullptr && (!aligned16(qt) || !aligned16(scales_t))) return FP8BQ_ERR_ALIGN;
  if (h != nullptr && !aligned16(h)) return FP8BQ_ERR_ALIGN;
  if (K % 128 != 0 || (qt != nullptr && M % 128 != 0)) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_rmsnorm_quant(x, M, K, ldx, gamma, eps, rstd, h, q, scales, qt, scales_t, fmt,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_rmsnorm_quantize_exact(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma, double eps,
                                 double* rstd, void* h, void* q, void* scales, void* qt, void* scales_t, int fmt,
                                 fp8bq_stream_t stream) {
  int st = check_quant_args(x, M, K, ldx, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (gamma == nullptr || rstd == nullptr) return FP8BQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0) || !std::isfinite(eps)) return FP8BQ_ERR_INVALID_ARG;  // finite, not negative
  if ((qt == nullptr) != (scales_t == nullptr)) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned16(gamma) || (reinterpret_cast<uintptr_t>(rstd) & 7u) != 0) return FP8BQ_ERR_ALIGN;
  if (qt != nullptr && (!aligned16(qt) || !aligned16(scales_t))) return FP8BQ_ERR_ALIGN;
  if (h != nullptr && !aligned16(h)) return FP8BQ_ERR_ALIGN;
  if (K % 128 != 0 || (qt != nullptr && M % 128 != 0)) return FP8BQ_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_rmsnorm_quant_exact(x, M, K, ldx, gamma, eps, rstd, h, q, scales, qt, scales_t,
                                                       fmt, reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw, void* q, void* scales,
                          int fmt, fp8bq_stream_t stream) {
  int st = check_quant_args(w, N, K, ldw, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  const fp8bq::QuantJob job{w, N, K, ldw, q, scales, nullptr, nullptr, true};
  return cuda_status(fp8bq::launch_quant_group(&job, 1, fmt, reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_quantize_group(const fp8bq_quant_job* jobs, int njobs, int fmt, fp8bq_stream_t stream) {
  if (jobs == nullptr || njobs < 1 || njobs > 8) return FP8BQ_ERR_INVALID_ARG;
  if (!valid_fmt(fmt)) return FP8BQ_ERR_INVALID_ARG;
  fp8bq::QuantJob jb[8];
  for (int i = 0; i < njobs; ++i) {
    const fp8bq_quant_job& j = jobs[i];
    const bool rows = j.kind == FP8BQ_QUANT_ACT || j.kind == FP8BQ_QUANT_ACT_DUAL || j.kind == FP8BQ_QUANT_WEIGHT;
    const bool cols = j.kind == FP8BQ_QUANT_ACT_T || j.kind == FP8BQ_QUANT_ACT_DUAL;
    if (!rows && !cols) return FP8BQ_ERR_INVALID_ARG;
    int st = FP8BQ_OK;
    if (rows && (st = check_quant_args(j.x, j.rows, j.cols, j.ldx, j.q, j.scales, fmt)) != FP8BQ_OK) return st;
    if (cols && (st = check_quant_args(j.x, j.rows, j.cols, j.ldx, j.qt, j.scales_t, fmt)) != FP8BQ_OK) return st;
    if (rows && j.cols % 128 != 0) return FP8BQ_ERR_SHAPE;
    if (cols && j.rows % 128 != 0) return FP8BQ_ERR_SHAPE;
    if (cols && j.cols % 8 != 0) return FP8BQ_ERR_ALIGN;
    jb[i] = fp8bq::QuantJob{j.x, j.rows, j.cols, j.ldx, rows ? j.q : nullptr, rows ? j.scales : nullptr,
                            cols ? j.qt : nullptr, cols ? j.scales_t : nullptr, j.kind == FP8BQ_QUANT_WEIGHT};
  }
  bool any = false;
  for (int i = 0; i < njobs; ++i) any = any || (jb[i].rows > 0 && jb[i].cols > 0);
  if (!any) return FP8BQ_OK;
  int st = device_ok();
  if (st != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_group(jb, njobs, fmt, reinterpret_cast<cudaStream_t>(stream)));
}

int fp8bq_gemm(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
               int64_t K, int64_t ldd, uint32_t flags, fp8bq_stream_t stream) {
  return fp8bq_gemm_ws(A, B, D, M, N, K, ldd, flags, nullptr, 0, stream);
}

int64_t fp8bq_gemm_workspace_bytes(void) {
  if (device_ok() != FP8BQ_OK) return -1;
  int sms = 0;
  if (fp8bq::device_sm_count(&sms) != cudaSuccess) return -1;
  return static_cast<int64_t>(sms / 2) * fp8bq::kWsSlotBytes;
}

int fp8bq_gemm_ws(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N, int64_t K,
                  int64_t ldd, uint32_t flags, void* workspace, int64_t workspace_bytes, fp8bq_stream_t stream) {
  if (workspace != nullptr && workspace_bytes < 0) return FP8BQ_ERR_INVALID_ARG;
  if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP8BQ_ERR_ALIGN;
  fp8bq::GemmProblem p;
  int st = fp8bq::validate_gemm(A, B, D, M, N, K, ldd, flags, &p);
  if (st != FP8BQ_OK) return st;
  p.ws = workspace;
  p.ws_bytes = workspace != nullptr ? workspace_bytes : 0;
  return fp8bq::run_gemm(p, reinterpret_cast<cudaStream_t>(stream));
}

int fp8bq_testing_gemm_ws_withhold(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
                                   int64_t K, int64_t ldd, uint32_t flags, void* workspace, int64_t workspace_bytes,
                                   int withhold_pair, int64_t wait_limit_ns, fp8bq_stream_t stream) {
  if (workspace == nullptr || workspace_bytes < 0 || withhold_pair < 0) return FP8BQ_ERR_INVALID_ARG;
  if (wait_limit_ns < 100000 || wait_limit_ns > 2000000000LL) return FP8BQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP8BQ_ERR_ALIGN;
  fp8bq::GemmProblem p;
  int st = fp8bq::validate_gemm(A, B, D, M, N, K, ldd, flags, &p);
  if (st != FP8BQ_OK) return st;
  p.ws = workspace;
  p.ws_bytes = workspace_bytes;
  p.withhold_cluster = withhold_pair;
  p.wait_limit_ns = static_cast<uint64_t>(wait_limit_ns);
  return fp8bq::run_gemm(p, reinterpret_cast<cudaStream_t>(stream));
}

int64_t fp8bq_row_scale_ld(int64_t rows) { return rows < 0 ? -1 : fp8bq::round_up128(rows); }

int64_t fp8bq_scales_bytes(int gran, int fmt, int64_t rows, int64_t contraction) {
  if (!valid_fmt(fmt) || rows < 0 || contraction < 0 || contraction % 128 != 0) return -1;
  const int64_t esz = fmt == FP8BQ_SCALE_FP32 ? 4 : 1;
  const int64_t nkb = contraction / 128;
  if (gran == FP8BQ_GRAN_ROW_1x128) return nkb * fp8bq::round_up128(rows) * esz;
  if (gran == FP8BQ_GRAN_ROW_1x32)
    return fmt == FP8BQ_SCALE_UE8M0 ? (contraction / 32) * fp8bq::round_up128(rows) : -1;
  if (gran == FP8BQ_GRAN_BLOCK_128x128) return nkb * ((rows + 127) / 128) * esz;
  return -1;
}

int fp8bq_check(fp8bq_stream_t stream) {
  int status = 0;
  cudaError_t e = fp8bq::read_and_clear_device_status(reinterpret_cast<cudaStream_t>(stream), &status);
  if (e != cudaSuccess) return cuda_status(e);
  return status != 0 ? FP8BQ_ERR_TIMEOUT : FP8BQ_OK;
}

int fp8bq_set_clock_counters(unsigned long long* counters) {
  if (counters != nullptr && (reinterpret_cast<uintptr_t>(counters) & 7u) != 0) return FP8BQ_ERR_ALIGN;
  int st = device_ok();
  if (st != FP8BQ_OK) return st;
  return cuda_status(fp8bq::set_clock_counters(counters));
}

int fp8bq_last_cuda_error(void) { return t_last_cuda_error; }

const char* fp8bq_status_string(int status) {
  switch (status) {
    case FP8BQ_OK: return "ok";
    case FP8BQ_ERR_INVALID_ARG: return "invalid argument";
    case FP8BQ_ERR_SHAPE: return "bad shape";
    case FP8BQ_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case FP8BQ_ERR_UNSUPPORTED: return "unsupported device or operand combination";
    case FP8BQ_ERR_CUDA: return "CUDA error";
    case FP8BQ_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int fp8bq_version(void) { return 100; }

}  // extern "C"
