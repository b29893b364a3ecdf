// testing.cu - the failure-detection hook of include/qlinear_testing.h.
#include "launch.h"
#include "sm100.cuh"
#include "../../include/qlinear_testing.h"

namespace ql {
namespace {

// One thread waits on a fresh mbarrier (phase 0 never completes: no thread
// arrives and no copy is issued) with the bounded wait of the pipelines.
__global__ void wait_timeout_kernel(int32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns))
    atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

}  // namespace
}  // namespace ql

extern "C" int ql_test_wait_timeout(int32_t* d_status, uint32_t limit_us, void* stream) {
  if (!d_status || limit_us < 1 || limit_us > 10000000u) return QL_ERR_ARG;
  ql::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      d_status, static_cast<unsigned long long>(limit_us) * 1000ull);
  ql::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}
