// gemm_noalloc.cu -- fp8bq_gemm_noalloc: the split-tile GEMM of fp8bq_gemm_ws
// with its workspace in a device array that belongs to this library, for
// callers that cannot allocate device memory themselves.
//
// Some callers have no way to hand the GEMM a workspace: code that may not
// call cudaMalloc because it can synchronize the whole device and stall the
// other streams (latency-bound serving loops), processes whose device memory
// is already held by another allocator (a framework's caching pool that has
// reserved nearly all of it, so a raw cudaMalloc fails), and plugin-style
// interfaces that pass a kernel its inputs and outputs and nothing else.
// For them the workspace lives in one file-scope __device__ array of fixed
// size, which every GPU that loads the library holds until the process
// exits.  The caller still passes the operands and D.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8bq.h"
#include "internal.h"

namespace {

// CTA pairs the array has a partial-sum slot for: 160 multiprocessors (a B200
// has 148, i.e. 74 pairs).  80 slots of 256 KB + 64 bytes: 20.98 MB.
constexpr int64_t kNoAllocPairs = 80;
constexpr int64_t kNoAllocBytes = kNoAllocPairs * fp8bq::kWsSlotBytes;

}  // namespace

// The workspace.  In host code this name is only a stand-in for the device
// object, not an address a kernel may use; its device address comes from
// cudaGetSymbolAddress (scratch_address below).
static __device__ __align__(256) unsigned char g_gemm_scratch[kNoAllocBytes];

namespace {

// Device address of g_gemm_scratch on the current device, looked up once
// per device (with that device current) and cached; nullptr on failure.
void* scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_gemm_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" int fp8bq_gemm_noalloc(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
                                  int64_t K, int64_t ldd, uint32_t flags, fp8bq_stream_t stream) {
  if (!A || !B || !D) return FP8BQ_ERR_INVALID_ARG;
  const int64_t need = fp8bq_gemm_workspace_bytes();  // one slot per CTA pair of this device
  if (need < 0) return FP8BQ_ERR_UNSUPPORTED;
  if (need > kNoAllocBytes) return FP8BQ_ERR_UNSUPPORTED;  // more CTA pairs than the array has slots for
  cudaError_t e = cudaSuccess;
  void* ws = scratch_address(&e);
  if (ws == nullptr) return FP8BQ_ERR_CUDA;
  // The flags after the slots must start at zero; the slots need not (a
  // piece stores its partial sum before its flag says so).  A completed
  // call leaves the flags zero, a failed one may not: clear them each time.
  const int64_t slots = need / fp8bq::kWsSlotBytes;
  e = cudaMemsetAsync(static_cast<unsigned char*>(ws) + slots * fp8bq::kWsTileBytes, 0,
                      static_cast<size_t>(slots * (fp8bq::kWsSlotBytes - fp8bq::kWsTileBytes)),
                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return FP8BQ_ERR_CUDA;
  return fp8bq_gemm_ws(A, B, D, M, N, K, ldd, flags, ws, need, stream);
}
