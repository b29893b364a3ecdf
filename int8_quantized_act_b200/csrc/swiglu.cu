// swiglu.cu - the SwiGLU gate of the MLP whose three projections run through
// this layer (w1 and w3 stacked as one call on the same input, w2 on h):
// h = silu(a) * b with silu(a) = a / (1 + e^-a).
//
// Forward: one kernel reads the stacked pre-activations [a | b] (the stacked
// projection's output) and writes the second projection's saved input
// directly, h quantized per row (int8 codes and s_h), so h itself never goes
// to memory.  Backward: one elementwise kernel turns dh (the second
// projection's input gradient) into [da | db], the stacked projection's
// output gradient.
//
// e^x is evaluated with fixed float32 steps so that codes decided through it
// are reproducible bit for bit: Cody and Waite's argument reduction (W. J.
// Cody, W. Waite, "Software Manual for the Elementary Functions", 1980),
// n = rint(x log2 e), r = (x - n C1) - n C2 with C1 = fl32(ln 2) and C2 the
// remainder, each a correctly rounded fused multiply-add; e^r by the Taylor
// series to degree 7 in Horner form (fused multiply-adds); times 2^n as the
// product of two exact powers of two.  x is clamped to [-104, 89] first.
// Groups of eight values whose a lie in [-16, 86] (|a| >= 2^-90) take a
// faster form with the same results (exp_fast2, and the correctly rounded
// division of divrn.cuh); others take these steps as written and the IEEE
// division.
#include <algorithm>

#include "divrn.cuh"
#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer

// e^x by the steps of the file comment, for every x (a NaN gives NaN).
// rint(y) for |y| < 2^22 is (y + 1.5*2^23) - 1.5*2^23, the integer n in the
// low bits of y + 1.5*2^23.
__device__ __forceinline__ float exp_ref(float x) {
  if (x != x) return x;
  const float xc = fminf(fmaxf(x, -104.0f), 89.0f);
  const float t = __fadd_rn(__fmul_rn(xc, 0x1.715476p+0f), kMagic);
  const float mn = __fsub_rn(kMagic, t);  // -rint(y)
  const int n = __float_as_int(t) - 0x4B400000;
  float r = __fmaf_rn(mn, 0x1.62e43p-1f, xc);
  r = __fmaf_rn(mn, -0x1.05c61p-29f, r);
  float p = 0x1.a01a02p-13f;
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
  p = __fmaf_rn(p, r, 0x1.111112p-7f);
  p = __fmaf_rn(p, r, 0x1.555556p-5f);
  p = __fmaf_rn(p, r, 0x1.555556p-3f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int a = n / 2;
  return __fmul_rn(__fmul_rn(p, __int_as_float((a + 127) << 23)), __int_as_float((n - a + 127) << 23));
}

// e^x of two values at once for -86 <= x <= 16, with packed f32x2
// multiplies and fused multiply-adds (each half one correctly rounded
// operation): the same result as exp_ref.  n lies in [-125, 23]: the Horner
// steps run on 2p (every coefficient doubled: each step scales exactly), and
// 2p * 2^(n-1), one multiply by a normal power of two, is p * 2^n with the
// one rounding of the two exact-then-rounded multiplies of exp_ref.  The rounding addition is
// scalar: a packed add of a packed product's result is fused into one fma by
// the code generator, which would skip the rounding of y.
__device__ __forceinline__ float2 exp_fast2(float2 x) {
  const float x0 = x.x, x1 = x.y;
  const float2 y = mul2(make_float2(x0, x1), make_float2(0x1.715476p+0f, 0x1.715476p+0f));
  const float t0 = __fadd_rn(y.x, kMagic), t1 = __fadd_rn(y.y, kMagic);
  const float2 mn = sub2(make_float2(kMagic, kMagic), make_float2(t0, t1));  // -rint(y)
  float2 r = fma2(mn, make_float2(0x1.62e43p-1f, 0x1.62e43p-1f), make_float2(x0, x1));
  r = fma2(mn, make_float2(-0x1.05c61p-29f, -0x1.05c61p-29f), r);
  float2 p = make_float2(0x1.a01a02p-12f, 0x1.a01a02p-12f);
  p = fma2(p, r, make_float2(0x1.6c16c2p-9f, 0x1.6c16c2p-9f));
  p = fma2(p, r, make_float2(0x1.111112p-6f, 0x1.111112p-6f));
  p = fma2(p, r, make_float2(0x1.555556p-4f, 0x1.555556p-4f));
  p = fma2(p, r, make_float2(0x1.555556p-2f, 0x1.555556p-2f));
  p = fma2(p, r, make_float2(1.0f, 1.0f));
  p = fma2(p, r, make_float2(2.0f, 2.0f));
  p = fma2(p, r, make_float2(2.0f, 2.0f));
  // 2^(n-1) = bits (n + 126) << 23, n = bits(t) - bits(1.5 * 2^23)
  const float s0 = __int_as_float((__float_as_int(t0) - (0x4B400000 - 126)) << 23);
  const float s1 = __int_as_float((__float_as_int(t1) - (0x4B400000 - 126)) << 23);
  return mul2(p, make_float2(s0, s1));
}

// Whether eight gate values take the fast steps: every a in [-16, 86] with
// |a| >= 2^-90 (no zero, NaN or infinity).  Then x = -a lies in [-86, 16],
// d = 1 + e^-a in [1, 2^24], and a / d is a normal float: the range of
// exp_fast2 and of the division's correction steps (divrn.cuh).
__device__ __forceinline__ bool fast_ok8(const float (&a)[8]) {
  float lo = fmin3_nan(a[0], a[1], a[2]), hi = fmax3_nan(a[0], a[1], a[2]);
  float mg = fmin3_nan(fabsf(a[0]), fabsf(a[1]), fabsf(a[2]));
  lo = fmin3_nan(lo, a[3], a[4]);
  hi = fmax3_nan(hi, a[3], a[4]);
  mg = fmin3_nan(mg, fabsf(a[3]), fabsf(a[4]));
  lo = fmin3_nan(lo, a[5], a[6]);
  hi = fmax3_nan(hi, a[5], a[6]);
  mg = fmin3_nan(mg, fabsf(a[5]), fabsf(a[6]));
  lo = fmin_nan(lo, a[7]);
  hi = fmax_nan(hi, a[7]);
  mg = fmin_nan(mg, fabsf(a[7]));
  return lo >= -16.0f && hi <= 86.0f && mg >= 0x1p-90f;
}

// d = 1 + e^-a and (with Q) q = a / d for eight values: the fast steps when
// fast_ok8 holds, else exp_ref and the IEEE division.  1 + e is a scalar
// addition (e comes from a packed multiply, see exp_fast2).  With R also
// y = 1/d.
template <bool R>
__device__ __forceinline__ void silu_parts8(const float (&a)[8], float (&q)[8], float (&y)[8]) {
  if (fast_ok8(a)) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float2 e = exp_fast2(make_float2(-a[k], -a[k + 1]));
      const float d0 = __fadd_rn(1.0f, e.x), d1 = __fadd_rn(1.0f, e.y);
      const float y0 = recip_rn(d0), y1 = recip_rn(d1);
      q[k] = div_rn(a[k], d0, y0);
      q[k + 1] = div_rn(a[k + 1], d1, y1);
      if (R) {
        y[k] = y0;
        y[k + 1] = y1;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float d = __fadd_rn(1.0f, exp_ref(-a[k]));
      q[k] = __fdiv_rn(a[k], d);
      if (R) y[k] = __fdiv_rn(1.0f, d);
    }
  }
}

constexpr int kGateThreads = 448;
constexpr int kGatePiece = 8;                          // columns per thread per piece
constexpr int kGateSpan = kGateThreads * kGatePiece;   // 3584 columns per piece

// One CTA per row of [a | b] (persistent over rows): thread t owns columns
// j * 3584 + 8t .. +7 of h for pieces j < P.  Each thread streams its own
// slots of the next row into shared memory with 16-byte asynchronous copies
// (cp.async, one commit group per piece): piece j of the next row is issued as
// soon as piece j of this row has been used, so the loads run under the rest
// of the row's arithmetic, and since a thread reads only what it copied, no
// barrier guards the slots.  The row maximum of |h| is a NaN-propagating max,
// reduced over the warps through shared memory; the codes are stored 8 at a
// time.  448 threads (14 warps), two CTAs per SM: d_ff = 14336 is exactly four
// pieces, and the 8 * P values of h a thread holds across its row fit the
// register budget of two CTAs per SM.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 8 values of a staged slot as float32.
__device__ __forceinline__ void slot8(uint32_t addr, const __nv_bfloat16*, float (&v)[8]) {
  const uint4 u = lds128(addr);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = __uint_as_float(w[e] << 16);
    v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void slot8(uint32_t addr, const float*, float (&v)[8]) {
  const uint4 u = lds128(addr), w = lds128(addr + 16);
  v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
  v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  v[4] = __uint_as_float(w.x); v[5] = __uint_as_float(w.y);
  v[6] = __uint_as_float(w.z); v[7] = __uint_as_float(w.w);
}

template <typename InT, int P>
__global__ void __launch_bounds__(kGateThreads, 2) swiglu_quant_kernel(
    const InT* __restrict__ ab, int64_t M, int F, int64_t ldab, int8_t* __restrict__ hq,
    int64_t ldh, float* __restrict__ sh, int32_t* __restrict__ status) {
  constexpr int E = kGatePiece * static_cast<int>(sizeof(InT));  // bytes of 8 values
  extern __shared__ __align__(16) uint8_t stage[];  // [P][a, b][kGateThreads][E]
  __shared__ uint32_t s_wmax[2][kGateThreads / 32];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const uint32_t base = smem_u32(stage);
  auto slot = [&](int j, int half) {
    return base + static_cast<uint32_t>(((j * 2 + half) * kGateThreads + t) * E);
  };
  // Piece j of row m into this thread's slots (nothing past the last row or
  // column), then one commit group either way.
  auto issue = [&](int64_t m, int j) {
    const int col = j * kGateSpan + t * kGatePiece;
    if (m < M && col < F) {
      const char* ra = reinterpret_cast<const char*>(ab + m * ldab + col);
      const char* rb = reinterpret_cast<const char*>(ab + m * ldab + F + col);
#pragma unroll
      for (int c = 0; c < E; c += 16) {
        cp_async16(slot(j, 0) + c, ra + c);
        cp_async16(slot(j, 1) + c, rb + c);
      }
    }
    cp_async_commit();
  };
  griddep_wait();  // [a | b] (a previous kernel's output) is visible from here
#pragma unroll
  for (int j = 0; j < P; ++j) issue(blockIdx.x, j);
  int par = 0;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x, par ^= 1) {
    const int64_t mn = m + gridDim.x;
    float h[P][kGatePiece];
    float mx0 = 0.0f, mx1 = 0.0f;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      // P groups are pending (this row's pieces j.., the next row's ..j-1):
      // the oldest, this row's piece j, has landed once at most P-1 remain.
      cp_async_wait<P - 1>();
      const int col = j * kGateSpan + t * kGatePiece;
      if (col < F) {
        float a8[8], b8[8];
        slot8(slot(j, 0), ab, a8);
        slot8(slot(j, 1), ab, b8);
        float s8[8], unused[8];
        silu_parts8<false>(a8, s8, unused);
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const float2 hv = mul2(make_float2(s8[k], s8[k + 1]), make_float2(b8[k], b8[k + 1]));
          h[j][k] = hv.x;
          h[j][k + 1] = hv.y;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) h[j][k] = 0.0f;
      }
      issue(mn, j);  // the slots are free: their values are in h[j]
#pragma unroll
      for (int k = 0; k < 8; k += 4) {
        mx0 = fmax3_nan(mx0, fabsf(h[j][k]), fabsf(h[j][k + 1]));
        mx1 = fmax3_nan(mx1, fabsf(h[j][k + 2]), fabsf(h[j][k + 3]));
      }
    }
    // Non-negative floats order like their bit patterns; NaN sorts last.
    uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fmax_nan(mx0, mx1)));
    if (lane == 0) s_wmax[par][warp] = mb;
    // Rows alternate between the two halves of s_wmax: this half is written
    // again only after the next row's barrier, which every thread reaches
    // after reading it here.
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kGateThreads / 32; ++w) mb = max(mb, s_wmax[par][w]);
    const float amax = __uint_as_float(mb);
    const float inv = mb == 0 ? 0.0f : 127.0f / amax;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const int col = j * kGateSpan + t * kGatePiece;
      if (col < F) {
        // products two at a time, the rounding adds one at a time
        uint32_t c[8];
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const float2 v = mul2(make_float2(h[j][k], h[j][k + 1]), make_float2(inv, inv));
          c[k] = __float_as_uint(__fadd_rn(v.x, kRneMagic));
          c[k + 1] = __float_as_uint(__fadd_rn(v.y, kRneMagic));
        }
        *reinterpret_cast<uint2*>(hq + m * ldh + col) =
            make_uint2(pack_codes(c[0], c[1], c[2], c[3]), pack_codes(c[4], c[5], c[6], c[7]));
      }
    }
    if (t == 0) {
      sh[m] = mb == 0 ? 0.0f : amax / 127.0f;
      if (mb >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
    }
  }
  griddep_launch_dependents();
  cp_async_wait<0>();  // the groups issued past the last row are empty
}

// [da | db] from [a | b] and dh, 8 columns per thread-step:
//   d = 1 + e^-a, sigma = 1/d, silu = a/d,
//   da = (dh * b) * (sigma * (1 + a * (1 - sigma))),  db = dh * silu.
template <typename InT, typename GT, typename OutT>
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const InT* __restrict__ ab, int64_t ldab,
                                                         const GT* __restrict__ dh, int64_t M,
                                                         int F, OutT* __restrict__ dab) {
  const int64_t per_row = F / 8;
  const int64_t total = M * per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t m = i / per_row;
    const int col = static_cast<int>(i - m * per_row) * 8;
    float a8[8], b8[8], g8[8], da[8], db[8];
    load8(ab + m * ldab + col, a8);
    load8(ab + m * ldab + F + col, b8);
    load8(dh + m * F + col, g8);
    float sg8[8], sl8[8];
    silu_parts8<true>(a8, sl8, sg8);  // silu = a/d, sigma = 1/d
    // ds = sigma * (1 + a * (1 - sigma)) scalar (its adds follow products);
    // the products with dh two at a time.
    float ds[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      ds[k] = __fmul_rn(sg8[k], __fadd_rn(1.0f, __fmul_rn(a8[k], __fsub_rn(1.0f, sg8[k]))));
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float2 g = make_float2(g8[k], g8[k + 1]);
      const float2 v = mul2(mul2(g, make_float2(b8[k], b8[k + 1])), make_float2(ds[k], ds[k + 1]));
      const float2 w = mul2(g, make_float2(sl8[k], sl8[k + 1]));
      da[k] = v.x;
      da[k + 1] = v.y;
      db[k] = w.x;
      db[k + 1] = w.y;
    }
    store8(dab + m * 2 * static_cast<int64_t>(F) + col, da);
    store8(dab + m * 2 * static_cast<int64_t>(F) + F + col, db);
  }
}

template <typename InT, int P>
cudaError_t gate_quant_t(const void* ab, int64_t M, int F, int64_t ldab, int8_t* hq, int64_t ldh,
                         float* sh, int32_t* st, cudaStream_t s) {
  auto kern = swiglu_quant_kernel<InT, P>;
  const size_t smem = static_cast<size_t>(P) * 2 * kGateThreads * kGatePiece * sizeof(InT);
  static int occ[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int per_sm = dev < 64 ? __atomic_load_n(&occ[dev], __ATOMIC_ACQUIRE) : 0;
  if (per_sm <= 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGateThreads, smem);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return e;
    }
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (dev < 64) __atomic_store_n(&occ[dev], per_sm, __ATOMIC_RELEASE);
  }
  const int grid = static_cast<int>(std::min<int64_t>(M, static_cast<int64_t>(device_info().sms) * per_sm));
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kGateThreads), smem, s,
                                   reinterpret_cast<const InT*>(ab), M, F, ldab, hq, ldh, sh, st);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <typename InT>
cudaError_t gate_quant_p(const void* ab, int64_t M, int F, int64_t ldab, int8_t* hq, int64_t ldh,
                         float* sh, int32_t* st, cudaStream_t s) {
  switch ((F + kGateSpan - 1) / kGateSpan) {
    case 1: return gate_quant_t<InT, 1>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 2: return gate_quant_t<InT, 2>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 3: return gate_quant_t<InT, 3>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 4: return gate_quant_t<InT, 4>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 5: return gate_quant_t<InT, 5>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 6: return gate_quant_t<InT, 6>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 7: return gate_quant_t<InT, 7>(ab, M, F, ldab, hq, ldh, sh, st, s);
    case 8: return gate_quant_t<InT, 8>(ab, M, F, ldab, hq, ldh, sh, st, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename GT>
cudaError_t gate_bwd_o(const void* ab, int64_t ldab, const void* dh, int64_t M, int F, void* dab,
                       int dabt, cudaStream_t s) {
  const int64_t total = M * (F / 8);
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(device_info().sms) * 8)));
  const InT* a = reinterpret_cast<const InT*>(ab);
  const GT* g = reinterpret_cast<const GT*>(dh);
  if (dabt == QL_BF16)
    swiglu_bwd_kernel<InT, GT, __nv_bfloat16><<<grid, 256, 0, s>>>(
        a, ldab, g, M, F, reinterpret_cast<__nv_bfloat16*>(dab));
  else
    swiglu_bwd_kernel<InT, GT, float><<<grid, 256, 0, s>>>(a, ldab, g, M, F,
                                                           reinterpret_cast<float*>(dab));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_swiglu_quant(const void* ab, int abt, int64_t M, int64_t F, int64_t ldab,
                                int8_t* hq, int64_t ldh, float* sh, int32_t* st, cudaStream_t s) {
  const cudaError_t e =
      abt == QL_BF16
          ? gate_quant_p<__nv_bfloat16>(ab, M, static_cast<int>(F), ldab, hq, ldh, sh, st, s)
          : gate_quant_p<float>(ab, M, static_cast<int>(F), ldab, hq, ldh, sh, st, s);
  count_launches(1);
  return e;
}

cudaError_t launch_swiglu_bwd(const void* ab, int abt, int64_t ldab, const void* dh, int dht,
                              int64_t M, int64_t F, void* dab, int dabt, cudaStream_t s) {
  const int f = static_cast<int>(F);
  cudaError_t e;
  if (abt == QL_BF16)
    e = dht == QL_BF16 ? gate_bwd_o<__nv_bfloat16, __nv_bfloat16>(ab, ldab, dh, M, f, dab, dabt, s)
                       : gate_bwd_o<__nv_bfloat16, float>(ab, ldab, dh, M, f, dab, dabt, s);
  else
    e = dht == QL_BF16 ? gate_bwd_o<float, __nv_bfloat16>(ab, ldab, dh, M, f, dab, dabt, s)
                       : gate_bwd_o<float, float>(ab, ldab, dh, M, f, dab, dabt, s);
  count_launches(1);
  return e;
}

}  // namespace ql
