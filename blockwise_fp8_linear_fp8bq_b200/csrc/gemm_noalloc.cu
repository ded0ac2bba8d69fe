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

// Device address of g_gemm_scratch in the context current on this thread.
// It is looked up (cudaGetSymbolAddress, with the device current) on the
// first call in each context and cached together with the context's
// identifier, so a new context on the same device (after cudaDeviceReset, or
// a context the caller created) is looked up again instead of being handed a
// stale address.  nullptr on failure, with the CUDA error in *err.
void* scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  static unsigned long long ctx[64] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = fp8bq::current_context_id();
  if (addr[dev] != nullptr && id != 0 && ctx[dev] == id) return addr[dev];
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_gemm_scratch);  // makes the device's context current if none is
  if (*err != cudaSuccess) return nullptr;
  addr[dev] = p;
  ctx[dev] = fp8bq::current_context_id();
  return p;
}

}  // namespace

extern "C" int fp8bq_gemm_noalloc(const fp8bq_operand* A, const fp8bq_operand* B, void* D, int64_t M, int64_t N,
                                  int64_t K, int64_t ldd, uint32_t flags, fp8bq_stream_t stream) {
  // every argument is checked before anything is queued on the stream
  fp8bq::GemmProblem p;
  int st = fp8bq::validate_gemm(A, B, D, M, N, K, ldd, flags, &p);
  if (st != FP8BQ_OK) return st;
  const int64_t need = fp8bq_gemm_workspace_bytes();  // one slot per CTA pair of this device
  if (need < 0) return FP8BQ_ERR_UNSUPPORTED;
  if (need > kNoAllocBytes) return FP8BQ_ERR_UNSUPPORTED;  // more CTA pairs than the array has slots for
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!p.acc_f32) {  // FP32 accumulation splits nothing and never touches the array
    cudaError_t e = cudaSuccess;
    void* ws = scratch_address(&e);
    if (ws == nullptr) return fp8bq::cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    // The flags after the slots must start at zero; the slots need not (a
    // piece stores its partial sum before its flag says so).  A completed
    // call leaves the flags zero, a failed one may not: clear them each time.
    const int64_t slots = need / fp8bq::kWsSlotBytes;
    e = cudaMemsetAsync(static_cast<unsigned char*>(ws) + slots * fp8bq::kWsTileBytes, 0,
                        static_cast<size_t>(slots * (fp8bq::kWsSlotBytes - fp8bq::kWsTileBytes)), s);
    if (e != cudaSuccess) return fp8bq::cuda_status(e);
    p.ws = ws;
    p.ws_bytes = need;
  }
  return fp8bq::run_gemm(p, s);
}
