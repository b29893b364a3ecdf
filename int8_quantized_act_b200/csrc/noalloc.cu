// noalloc.cu - qlinear_bwd_dx_noalloc: the input-gradient call for callers
// that cannot allocate device memory (see include/qlinear.h).  Its scratch is
// a fixed array in this file's device image instead of a caller workspace.
#include <mutex>

#include "launch.h"
#include "../../include/qlinear.h"

namespace {

// The scratch of every qlinear_bwd_dx_noalloc call.  In host code this name is
// only a handle for the runtime: handing it to a kernel would pass a host
// address, so the host takes the device address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct DeviceScratch {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};

DeviceScratch g_scratch[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceScratch& d = g_scratch[dev];
  std::call_once(d.once, [&d] { d.err = cudaGetSymbolAddress(&d.ptr, g_noalloc_scratch); });
  if (d.err != cudaSuccess) return d.err;
  *out = d.ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" int qlinear_bwd_dx_noalloc(const void* dy, int dyt, int64_t M, int64_t N,
                                      const int8_t* wq, const float* sw, int64_t K,
                                      int hadamard_block, void* dx, int dxt, int32_t* d_status,
                                      void* stream) {
  if (M >= 0 && N >= 0 && K >= 0 &&
      qlinear_workspace_bytes(M, N, K, hadamard_block) > QL_NOALLOC_SCRATCH_BYTES)
    return QL_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return QL_ERR_CUDA;
  return qlinear_bwd_dx(dy, dyt, M, N, wq, sw, K, hadamard_block, dx, dxt, scratch,
                        QL_NOALLOC_SCRATCH_BYTES, d_status, stream);
}
