// noalloc.cu - qlinear_bwd_dx_noalloc: the input-gradient call for callers
// that cannot allocate device memory (see include/qlinear.h).  Its scratch is
// a fixed array in this file's device image instead of a caller workspace.
#include <atomic>

#include "launch.h"
#include "../../include/qlinear.h"

namespace {

// The scratch of every qlinear_bwd_dx_noalloc call.  In host code this name is
// only a handle for the runtime: handing it to a kernel would pass a host
// address, so the host takes the device address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of the array, per device; null until a lookup succeeded.
std::atomic<void*> g_scratch[kMaxDevices];

// Device address of the scratch array on the current device.  The lookup runs
// with that device current and only a successful one is kept, so a lookup
// that failed (for example because the library's device code could not be
// loaded while memory was short) is tried again by the next call.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();  // clear the failed call's error for later calls
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    // Two threads may both look it up; they store the same address.
    g_scratch[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" int qlinear_bwd_dx_noalloc(const void* dy, int dyt, int64_t M, int64_t N,
                                      const int8_t* wq, const float* sw, int64_t K,
                                      int hadamard_block, void* dx, int dxt, int32_t* d_status,
                                      void* stream) {
  // The argument and shape checks of qlinear_bwd_dx first, so both calls
  // return the same code for the same mistake; then the capacity.
  bool noop = false;
  const int pre = ql::check_bwd_dx_args(dy, dyt, M, N, wq, sw, K, hadamard_block, dx, dxt,
                                        d_status, &noop);
  if (pre != QL_OK || noop) return pre;
  if (qlinear_workspace_bytes(M, N, K, hadamard_block) > QL_NOALLOC_SCRATCH_BYTES)
    return QL_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return QL_ERR_CUDA;
  return qlinear_bwd_dx(dy, dyt, M, N, wq, sw, K, hadamard_block, dx, dxt, scratch,
                        QL_NOALLOC_SCRATCH_BYTES, d_status, stream);
}
