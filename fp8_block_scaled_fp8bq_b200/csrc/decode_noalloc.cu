// Decode-shaped linear that allocates nothing and takes no workspace.
//
// fp8bq_gemm_decode needs a device workspace (the quantized activation, its
// scales and the split-K partials) that the caller allocates.  Some callers
// cannot allocate device memory when they call: a host program written in C
// or Fortran that links this library without a framework's memory pool, or a
// serving loop that must not allocate once it is running (a fixed memory
// budget, or another library owns the device's memory).  This entry point
// gives them the same operation with its scratch in a file-scope device array
// of fixed size.  The array exists on every GPU that loads the library, for
// the life of the process.
#include <mutex>

#include "internal.h"

namespace fp8bq {
namespace {

// Largest workspace this entry point can serve (32 MiB per device).  Enough
// for every decode shape up to M = 256 tokens with K <= 14336 and N <= 28672.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch per device.  In host code the array's
// name only stands in for the symbol, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
void *g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

fp8bq_status scratch_for_current_device(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return FP8BQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FP8BQ_OK;
}

}  // namespace
}  // namespace fp8bq

using namespace fp8bq;

extern "C" {

fp8bq_status fp8bq_gemm_decode_noalloc(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw,
                                       void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                                       void *stream) {
  // Every argument check of fp8bq_gemm_decode comes first (so a bad pointer
  // or an unsupported size is reported as such), then the shapes whose
  // workspace would not fit in the fixed scratch are refused; nothing runs
  // before these checks pass.
  bool work = false;
  fp8bq_status st = check_decode_args(x, ldx, qw, ldw, sw, y, ldy, M, N, K, mode, &work);
  if (st != FP8BQ_OK || !work) return st;
  if (K > 0 && fp8bq_gemm_decode_workspace_size(M, N, K) > kNoAllocScratchBytes)
    return FP8BQ_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != FP8BQ_OK) return st;
  return fp8bq_gemm_decode(x, ldx, qw, ldw, sw, y, ldy, M, N, K, mode, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
