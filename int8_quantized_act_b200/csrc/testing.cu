// testing.cu - the hooks of include/qlinear_testing.h: the failure-detection
// wait and the gate's division steps.
#include <algorithm>

#include "divrn.cuh"
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

__global__ void divrn_kernel(const float* __restrict__ a, const float* __restrict__ d, int64_t n,
                             float* __restrict__ q, float* __restrict__ y) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float av = a[i], dv = d[i];
    const bool ok = div_rn_ok(av, dv) || div_rn_ok_wide(av, dv);
    const float r = ok ? recip_rn(dv) : __fdiv_rn(1.0f, dv);
    y[i] = r;
    q[i] = ok ? div_rn(av, dv, r) : __fdiv_rn(av, dv);
  }
}

__global__ void sqrtrn_kernel(const float* __restrict__ v, int64_t n, float* __restrict__ s0,
                              float* __restrict__ s1) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float x = v[i];
    const bool ok = sqrt_rn_ok(x);
    s0[i] = ok ? sqrt_rn_t<false>(x) : __fsqrt_rn(x);
    s1[i] = ok ? sqrt_rn_t<true>(x) : __fsqrt_rn(x);
  }
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

extern "C" int ql_test_divrn(const float* a, const float* d, int64_t n, float* q, float* y,
                             void* stream) {
  if (n < 0 || (n > 0 && (!a || !d || !q || !y))) return QL_ERR_ARG;
  if (n == 0) return QL_OK;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
  ql::divrn_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      a, d, n, q, y);
  ql::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

extern "C" int ql_test_sqrtrn(const float* v, int64_t n, float* s_plain, float* s_refined,
                              void* stream) {
  if (n < 0 || (n > 0 && (!v || !s_plain || !s_refined))) return QL_ERR_ARG;
  if (n == 0) return QL_OK;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
  ql::sqrtrn_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      v, n, s_plain, s_refined);
  ql::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}
