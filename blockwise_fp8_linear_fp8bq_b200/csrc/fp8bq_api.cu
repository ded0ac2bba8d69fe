// fp8bq_api.cu -- the C ABI declared in include/fp8bq.h: argument checks,
// status codes and dispatch to the kernels.  Nothing here allocates device
// memory or synchronizes, except fp8bq_check().
#include <cuda_runtime.h>

#include <cstdint>

#include "fp8bq.h"
#include "internal.h"

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FP8BQ_OK;
  t_last_cuda_error = static_cast<int>(e);
  return FP8BQ_ERR_CUDA;
}

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
int convert_operand(const fp8bq_operand* op, int64_t rows, int64_t K, bool is_a, int fmt,
                    fp8bq::GemmOperand* out) {
  if (!op || !op->data) return FP8BQ_ERR_INVALID_ARG;
  if (op->dtype != FP8BQ_E4M3 && op->dtype != FP8BQ_BF16) return FP8BQ_ERR_INVALID_ARG;
  if (op->gran != FP8BQ_GRAN_ROW_1x128 && op->gran != FP8BQ_GRAN_BLOCK_128x128 &&
      op->gran != FP8BQ_GRAN_ROW_1x32)
    return FP8BQ_ERR_INVALID_ARG;
  if (op->fmt != fmt) return FP8BQ_ERR_UNSUPPORTED;
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
  int st = check_quant_args(gu, M, 2 * F, ldgu, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if ((qt == nullptr) != (scales_t == nullptr)) return FP8BQ_ERR_INVALID_ARG;
  if (qt != nullptr && (!aligned16(qt) || !aligned16(scales_t))) return FP8BQ_ERR_ALIGN;
  if (h != nullptr && !aligned16(h)) return FP8BQ_ERR_ALIGN;
  if (F % 128 != 0 || (qt != nullptr && M % 128 != 0)) return FP8BQ_ERR_SHAPE;
  if (M == 0 || F == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_swiglu_quant(gu, M, F, ldgu, h, q, scales, qt, scales_t, fmt,
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

int fp8bq_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw, void* q, void* scales,
                          int fmt, fp8bq_stream_t stream) {
  int st = check_quant_args(w, N, K, ldw, q, scales, fmt);
  if (st != FP8BQ_OK) return st;
  if (K % 128 != 0) return FP8BQ_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8BQ_OK;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  return cuda_status(fp8bq::launch_quant_weight(w, N, K, ldw, q, scales, fmt,
                                                reinterpret_cast<cudaStream_t>(stream)));
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
  if (!A || !B || !D) return FP8BQ_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(FP8BQ_GEMM_ACCUMULATE_F32)) != 0) return FP8BQ_ERR_INVALID_ARG;
  const bool acc = (flags & FP8BQ_GEMM_ACCUMULATE_F32) != 0;
  if (!valid_fmt(A->fmt)) return FP8BQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0 || ldd < N) return FP8BQ_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return FP8BQ_ERR_SHAPE;
  if (!aligned16(D) || ldd % 8 != 0) return FP8BQ_ERR_ALIGN;
  if (workspace != nullptr && workspace_bytes < 0) return FP8BQ_ERR_INVALID_ARG;
  if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP8BQ_ERR_ALIGN;
  fp8bq::GemmProblem p;
  int st = convert_operand(A, M, K, true, A->fmt, &p.a);
  if (st != FP8BQ_OK) return st;
  st = convert_operand(B, N, K, false, A->fmt, &p.b);
  if (st != FP8BQ_OK) return st;
  if (p.a.mx != p.b.mx) return FP8BQ_ERR_UNSUPPORTED;  // MX blocks on both operands or neither
  // FP32 accumulation is built for the weight-gradient layout only
  if (acc && (p.a.bf16 || !p.a.row_groups || !p.b.row_groups || !p.b.k_major)) return FP8BQ_ERR_UNSUPPORTED;
  if ((st = device_ok()) != FP8BQ_OK) return st;
  p.d = D;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ldd = ldd;
  p.fmt = A->fmt;
  p.acc_f32 = acc;
  p.ws = workspace;
  p.ws_bytes = workspace != nullptr ? workspace_bytes : 0;
  bool unsupported = false;
  cudaError_t e = fp8bq::launch_gemm(p, reinterpret_cast<cudaStream_t>(stream), &unsupported);
  if (unsupported) return FP8BQ_ERR_UNSUPPORTED;
  return cuda_status(e);
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
