// muon.cu - MuonAuxAdamW for the layer's int8 weights (mini_trainer
// "docs/quantized-training.md", feature table row "Optimizers", which names
// it; the method is the published Muon optimizer of Jordan et al., 2024):
//   M' = beta*M + (1-beta)*G,   U = (1-beta)*G + beta*M'          (Nesterov)
//   X = U (or U^T when N > K), X /= ||X||_F + 1e-7, then 5 quintic
//   Newton-Schulz steps  A = X X^T,  B = b A + c A A,  X = a X + B X
//   w' = w (1 - lr wd) - lr max(1, N/K)^0.5 O  (O = X, back in [N, K]),
//   then the layer's Philox-keyed stochastic requantization per row.
// The Newton-Schulz products run on the tcgen05 bf16 GEMM (float32
// accumulation, bf16 operands as in the published method); X is kept in both
// layouts so that every product reads K-major operands: A = X X^T from X and
// X, A A = A A^T (A is symmetric), B X from B and X^T.  The step
// X' = a X + B X and its transpose are written by the B X product's epilogue
// (GemmEpilogue::ns_x); the other elementwise steps (momentum with ||U||^2,
// normalization, b A + c A A) are the kernels below; the requantization is
// update_sr.cu's.
// The float parameters of MuonAuxAdamW (biases, magnitudes) take AdamW:
// qadamw_vector.
#include <cuda_bf16.h>

#include <algorithm>

#include "launch.h"
#include "rowops.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;

// M' = beta*M + omb*G; U = omb*G + beta*M' (float32, in this order); the sum
// of U^2 in float64 (one atomic per block).
__global__ void __launch_bounds__(256) muon_momentum_kernel(const float* __restrict__ G,
                                                            float* __restrict__ M, int64_t n4,
                                                            float beta, float omb,
                                                            double* __restrict__ sumsq) {
  __shared__ double s_part[8];
  double acc = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 g = __ldcs(reinterpret_cast<const float4*>(G) + i);
    const float4 m = reinterpret_cast<const float4*>(M)[i];
    const float gg[4] = {g.x, g.y, g.z, g.w}, mm[4] = {m.x, m.y, m.z, m.w};
    float mo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      mo[e] = __fadd_rn(__fmul_rn(beta, mm[e]), __fmul_rn(omb, gg[e]));
      const float u = __fadd_rn(__fmul_rn(omb, gg[e]), __fmul_rn(beta, mo[e]));
      acc += static_cast<double>(u) * static_cast<double>(u);
    }
    reinterpret_cast<float4*>(M)[i] = make_float4(mo[0], mo[1], mo[2], mo[3]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += s_part[w];
    atomicAdd(sumsq, t);
  }
}

// One 64 x 64 tile of a row-major [rows, cols] float-valued matrix (rows,
// cols multiples of 8) written as bf16 into out [rows, cols] (if given) and
// transposed into out_t [cols, rows].  load(i, j, v) gives the 8 values at
// row i, columns j..j+7.  Thread t computes rows t/8 and t/8 + 32, columns
// 8(t%8)..+7 (16-byte stores; the thread that reads an element is the one
// that writes it in out), then writes rows t/8 and t/8 + 32 of the
// transposed tile, 8 values gathered from a column of the shared tile (rows
// padded to 66 values: conflict-free), 16 bytes a store.
template <typename F>
__device__ __forceinline__ void transpose64(int64_t rows, int64_t cols, int64_t r0, int64_t c0,
                                            F&& load, __nv_bfloat16* __restrict__ out,
                                            __nv_bfloat16* __restrict__ out_t,
                                            __nv_bfloat16 (*tile)[66]) {
  const int t = threadIdx.x, tr = t >> 3, tc = (t & 7) * 8;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int lr = tr + 32 * h;
    const int64_t i = r0 + lr, j = c0 + tc;
    if (i < rows && j < cols) {
      float v[8];
      load(i, j, v);
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat16 b0 = __float2bfloat16_rn(v[2 * k]);
        const __nv_bfloat16 b1 = __float2bfloat16_rn(v[2 * k + 1]);
        tile[lr][tc + 2 * k] = b0;
        tile[lr][tc + 2 * k + 1] = b1;
        o[k] = static_cast<uint32_t>(__bfloat16_as_ushort(b0)) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(b1)) << 16);
      }
      if (out) *reinterpret_cast<uint4*>(out + i * cols + j) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int lc = tr + 32 * h;                // row of the transposed tile
    const int64_t ci = c0 + lc, rj = r0 + tc;  // out_t [cols, rows]
    if (ci < cols && rj < rows) {
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o[k] = static_cast<uint32_t>(__bfloat16_as_ushort(tile[tc + 2 * k][lc])) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(tile[tc + 2 * k + 1][lc])) << 16);
      *reinterpret_cast<uint4*>(out_t + ci * rows + rj) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void load8f(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}


// X0 = bf16(U / (||U||_F + 1e-7)) with U recomputed from G and the new M
// (the same float32 operations as muon_momentum_kernel), written as X [r, c]
// and X^T [c, r], where X = U when N <= K (r = N) and X = U^T otherwise.
__global__ void __launch_bounds__(256) ns_init_kernel(const float* __restrict__ G,
                                                      const float* __restrict__ M, int64_t N,
                                                      int64_t K, float beta, float omb,
                                                      const double* __restrict__ sumsq,
                                                      __nv_bfloat16* __restrict__ X,
                                                      __nv_bfloat16* __restrict__ Xt) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][66];
  const float inv = static_cast<float>(1.0 / (sqrt(*sumsq) + 1e-7));
  const int64_t tiles_c = (K + 63) / 64, tiles = ((N + 63) / 64) * tiles_c;
  const bool tr = N > K;
  auto load = [&](int64_t r, int64_t c, float (&v)[8]) {
    float g[8], m[8];
    load8f(G + r * K + c, g);
    load8f(M + r * K + c, m);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      v[k] = __fmul_rn(__fadd_rn(__fmul_rn(omb, g[k]), __fmul_rn(beta, m[k])), inv);
  };
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int64_t r0 = (t / tiles_c) * 64, c0 = (t % tiles_c) * 64;
    // U [N, K] row-major; its transpose [K, N].  X is U or U^T.
    transpose64(N, K, r0, c0, load, tr ? Xt : X, tr ? X : Xt, tile);
  }
}

// AdamW on a float32 vector: the per-element arithmetic of the int8 update.
__global__ void __launch_bounds__(256) adamw_vector_kernel(float* __restrict__ p,
                                                           const float* __restrict__ g,
                                                           float* __restrict__ m,
                                                           float* __restrict__ v, int64_t n,
                                                           UpdateConsts c,
                                                           int32_t* __restrict__ status) {
  bool bad = false;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    float mm = m[i], vv = v[i];
    const float gi = g[i];
    const float w1 = p[i] * c.a;
    const float mn = c.b1 * mm + c.omb1 * gi;
    const float vn = c.b2 * vv + c.omb2 * (gi * gi);
    const float den = sqrtf(vn) * c.rbc2 + c.eps;
    const float w = w1 - c.st * (mn / den);
    m[i] = mn;
    v[i] = vn;
    p[i] = w;
    bad |= !isfinite(w);
  }
  if (bad) atomicOr(status, 1 << QL_ERR_NONFINITE);
}

int grid_for(int64_t items, int per_sm) {
  const int64_t cap = static_cast<int64_t>(device_info().sms) * per_sm;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, cap)));
}

}  // namespace

MuonLayout muon_layout(int64_t N, int64_t K) {
  MuonLayout L;
  const int64_t r = std::min(N, K), c = std::max(N, K);
  auto a256 = [](int64_t x) { return (x + 255) / 256 * 256; };
  int64_t off = 0;
  L.sumsq = off; off += 256;
  L.X = off;     off += a256(2 * r * c);
  L.Xt = off;    off += a256(2 * r * c);
  L.Xt2 = off;   off += a256(2 * r * c);
  L.A = off;     off += a256(2 * r * r);
  L.Bm = off;    off += a256(2 * r * r);
  L.total = off;
  return L;
}

cudaError_t launch_muon_orthogonalize(const float* grad, float* mom, int64_t N, int64_t K,
                                      float beta, int steps, void* O, void* ws, int32_t* status,
                                      cudaStream_t s) {
  const MuonLayout L = muon_layout(N, K);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  double* sumsq = reinterpret_cast<double*>(w + L.sumsq);
  auto* X = reinterpret_cast<__nv_bfloat16*>(w + L.X);
  auto* Xt = reinterpret_cast<__nv_bfloat16*>(w + L.Xt);
  auto* A = reinterpret_cast<__nv_bfloat16*>(w + L.A);
  auto* Bm = reinterpret_cast<__nv_bfloat16*>(w + L.Bm);
  __nv_bfloat16* xt_in = Xt;  // X^T as the B X product reads it
  __nv_bfloat16* xt_out = reinterpret_cast<__nv_bfloat16*>(w + L.Xt2);
  const int64_t r = std::min(N, K), c = std::max(N, K);
  const float omb = static_cast<float>(1.0 - static_cast<double>(beta));
  cudaError_t e = cudaMemsetAsync(sumsq, 0, sizeof(double), s);
  if (e != cudaSuccess) return e;
  muon_momentum_kernel<<<grid_for(N * K / 4, 8), 256, 0, s>>>(grad, mom, N * K / 4, beta, omb, sumsq);
  ns_init_kernel<<<grid_for(((N + 63) / 64) * ((K + 63) / 64) * 256, 8), 256, 0, s>>>(
      grad, mom, N, K, beta, omb, sumsq, X, Xt);
  count_launches(2);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int it = 0; it < steps; ++it) {
    // A = X X^T and B = b A + c (A A) are symmetric: the GEMM computes their
    // upper 256 x 256 tiles and its epilogue also writes each strictly upper
    // tile transposed into the lower one (exactly symmetric results); B is
    // formed in the A A product's epilogue from A and the float32
    // accumulator.
    GemmEpilogue ep;
    ep.out = A;
    ep.out_bf16 = 1;
    ep.ldo = r;
    ep.ns_mirror = 1;
    bool upper = true;
    if ((e = launch_gemm_bf16(X, c, X, c, r, r, c, ep, status, s, &upper)) != cudaSuccess) return e;  // A = X X^T
    ep.out = Bm;
    ep.ns_x = A;
    ep.ns_a = kNsB;
    ep.ns_c = kNsC;
    upper = true;
    if ((e = launch_gemm_bf16(A, r, A, r, r, r, r, ep, status, s, &upper)) != cudaSuccess) return e;  // b A + c A A
    // X' = a X + B X in the product's epilogue: X' over X (in place: each
    // element is read and written by the same thread, and X is not an
    // operand of this product) and X'^T into the other X^T buffer (the one
    // read here is the product's B operand).  The last step writes the
    // [N, K]-shaped layout (X'^T when N > K) into O.
    __nv_bfloat16* xo = X;
    __nv_bfloat16* xto = xt_out;
    if (it == steps - 1) {
      if (N > K) xto = reinterpret_cast<__nv_bfloat16*>(O);
      else xo = reinterpret_cast<__nv_bfloat16*>(O);
    }
    ep.out = xo;
    ep.ldo = c;
    ep.ns_mirror = 0;
    ep.ns_x = X;
    ep.ns_xt = xto;
    ep.ns_ldt = r;
    ep.ns_a = kNsA;
    ep.ns_c = 1.0f;
    if ((e = launch_gemm_bf16(Bm, r, xt_in, r, r, c, r, ep, status, s)) != cudaSuccess) return e;  // B X
    std::swap(xt_in, xt_out);
  }
  return cudaSuccess;
}

cudaError_t launch_adamw_vector(float* p, const float* g, float* m, float* v, int64_t n,
                                const UpdateConsts& c, int32_t* status, cudaStream_t s) {
  adamw_vector_kernel<<<grid_for(n, 8), 256, 0, s>>>(p, g, m, v, n, c, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ql
