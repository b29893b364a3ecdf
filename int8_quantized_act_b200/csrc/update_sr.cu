// update_sr.cu - fused optimizer step + stochastic requantization of int8
// weight rows (mini_trainer "docs/quantized-training.md": the paragraph after
// the feature table - updates requantize the represented weights
// stochastically in CUDA row kernels, with no floating master weight; feature
// table rows "Optimizers" and "Row-wise weight normalization").
//
// Each row is read from HBM once: codes, gradient and moments in, new moments
// out, while the updated float row waits in shared memory for the row max;
// the new scale follows from a max reduction over the row; then every
// 4-element chunk draws one Philox4x32-10 block and writes 4 stochastically
// rounded codes.  Rows up to ~8.8K elements are staged whole by the
// bulk-copy engine, one row per CTA (update_sr_staged_kernel); longer rows
// stream through a ring of row pieces in one persistent CTA per SM
// (update_sr_ring_kernel).  The row-wise weight-norm variant stages its
// codes and gradient (update_sr_wn_staged_kernel) and keeps 16-element groups
// only for the pinned order of its direction-gradient reduction.  The Muon
// step (update_sr_dir_kernel) takes a precomputed update direction.  Bytes
// per element: AdamW 22 (1+4+4+4 in, 1+4+4 out), SGD 6.
#include <cuda_runtime.h>

#include <algorithm>

#include "divrn.cuh"
#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

__device__ __forceinline__ float adamw(const UpdateConsts& c, float w, float g, float& m,
                                       float& v) {
  const float w1 = w * c.a;
  const float mn = c.b1 * m + c.omb1 * g;
  const float vn = c.b2 * v + c.omb2 * (g * g);
  const float den = sqrtf(vn) * c.rbc2 + c.eps;
  m = mn;
  v = vn;
  return w1 - c.st * (mn / den);
}

// The same step on four elements.  The square root and the division are the
// correctly rounded steps of divrn.cuh when the constants allow it (c.fast)
// and every v' lies in [2^-100, 2^100] and every m' in +-[2^-66, 2^60]: then
// den = sqrt(v')*rbc2 + eps lies in [2^-60, 2^60] and m'/den is a normal
// float.  Otherwise the IEEE operations; the results are the same bits.
// Those steps run on pairs of elements (f32x2 multiplies and fused
// multiply-adds; each half is the scalar IEEE operation).  A product that
// is added to something stays a scalar multiply: a packed multiply feeding
// a packed add can be compiled into one fused multiply-add.
__device__ __forceinline__ void adamw4(const UpdateConsts& c, const float (&w)[4],
                                      const float (&g)[4], float (&m)[4], float (&v)[4],
                                      float (&out)[4]) {
  float mn[4], vn[4], q[4];
#pragma unroll
  for (int h = 0; h < 4; h += 2) {
    const float2 gg = mul2(make_float2(g[h], g[h + 1]), make_float2(g[h], g[h + 1]));
    const float gs[2] = {gg.x, gg.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      mn[h + e] = __fadd_rn(__fmul_rn(c.b1, m[h + e]), __fmul_rn(c.omb1, g[h + e]));
      vn[h + e] = __fadd_rn(__fmul_rn(c.b2, v[h + e]), __fmul_rn(c.omb2, gs[e]));
    }
  }
  const float vlo = fmin_nan(fmin3_nan(vn[0], vn[1], vn[2]), vn[3]);
  const float vhi = fmax_nan(fmax3_nan(vn[0], vn[1], vn[2]), vn[3]);
  const float mlo = fmin_nan(fmin3_nan(fabsf(mn[0]), fabsf(mn[1]), fabsf(mn[2])), fabsf(mn[3]));
  const float mhi = fmax_nan(fmax3_nan(fabsf(mn[0]), fabsf(mn[1]), fabsf(mn[2])), fabsf(mn[3]));
  if (c.fast && vlo >= 0x1p-100f && vhi <= 0x1p+100f && mlo >= 0x1p-66f && mhi <= 0x1p+60f) {
#pragma unroll
    for (int h = 0; h < 4; h += 2) {
      // sqrt_rn_t<false> (v' > 0 here), then recip_rn and div_rn, two at a time
      const float2 vv = make_float2(vn[h], vn[h + 1]);
      const float2 z = make_float2(rsqrt_approx(vv.x), rsqrt_approx(vv.y));
      const float2 g0 = mul2(vv, z);
      const float2 hz = mul2(make_float2(0.5f, 0.5f), z);
      const float2 rs = fma2(make_float2(-g0.x, -g0.y), g0, vv);
      const float2 sq = fma2(rs, hz, g0);
      const float d0 = __fadd_rn(__fmul_rn(sq.x, c.rbc2), c.eps);
      const float d1 = __fadd_rn(__fmul_rn(sq.y, c.rbc2), c.eps);
      const float2 nd = make_float2(-d0, -d1);
      const float2 y0 = make_float2(rcp_approx(d0), rcp_approx(d1));
      const float2 ey = fma2(nd, y0, make_float2(1.0f, 1.0f));
      const float2 y = fma2(y0, ey, y0);
      const float2 mm = make_float2(mn[h], mn[h + 1]);
      const float2 q0 = mul2(mm, y);
      const float2 rq = fma2(nd, q0, mm);
      const float2 qq = fma2(rq, y, q0);
      q[h] = qq.x;
      q[h + 1] = qq.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) q[e] = mn[e] / (sqrtf(vn[e]) * c.rbc2 + c.eps);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    out[e] = __fsub_rn(__fmul_rn(w[e], c.a), __fmul_rn(c.st, q[e]));
    m[e] = mn[e];
    v[e] = vn[e];
  }
}

// The codes of a 4-element chunk w under the scale inverse inv with the
// chunk's Philox words rn: for v = w[e] * inv and u24 = rn[e] >> 8, floor(v)
// + 1 with probability frac(v), decided by u24 < frac * 2^24, clamped to
// [-127, 127]; the integer-valued result plus 1.5 * 2^23 (exact below 2^22
// in magnitude) holds the int8 code in its low byte, and the four low bytes
// are packed.  The products w * inv stay scalar (their difference with the
// floor is taken next); frac * 2^24, f + 1 and the rounding add run two at
// a time.
__device__ __forceinline__ uint32_t sr_codes4(float4 w, float inv, uint4 rn) {
  const float v[4] = {__fmul_rn(w.x, inv), __fmul_rn(w.y, inv), __fmul_rn(w.z, inv),
                      __fmul_rn(w.w, inv)};
  const uint32_t u[4] = {rn.x >> 8, rn.y >> 8, rn.z >> 8, rn.w >> 8};
  float f[4], fr[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[e] = floorf(v[e]);
    fr[e] = __fsub_rn(v[e], f[e]);
  }
  const float2 s24 = make_float2(16777216.0f, 16777216.0f), one = make_float2(1.0f, 1.0f);
  const float2 t01 = mul2(make_float2(fr[0], fr[1]), s24), t23 = mul2(make_float2(fr[2], fr[3]), s24);
  const float2 u01 = add2(make_float2(f[0], f[1]), one), u23 = add2(make_float2(f[2], f[3]), one);
  const float t[4] = {t01.x, t01.y, t23.x, t23.y}, f1[4] = {u01.x, u01.y, u23.x, u23.y};
  float r[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    r[e] = (__uint2float_rn(u[e]) < t[e]) ? f1[e] : f[e];
    r[e] = fminf(fmaxf(r[e], -127.0f), 127.0f);
  }
  const float2 mg = make_float2(kRneMagic, kRneMagic);
  const float2 c01 = add2(make_float2(r[0], r[1]), mg), c23 = add2(make_float2(r[2], r[3]), mg);
  return pack_codes(__float_as_uint(c01.x), __float_as_uint(c01.y), __float_as_uint(c23.x),
                    __float_as_uint(c23.y));
}

__device__ __forceinline__ void load16f(const float* p, float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 a = reinterpret_cast<const float4*>(p)[i];
    v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
  }
}

__device__ __forceinline__ int code_at(const uint4& q, int i) {
  const uint32_t w = (&q.x)[i >> 2];
  return static_cast<int>(static_cast<int8_t>((w >> (8 * (i & 3))) & 0xFFu));
}

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of two
// 32x32->64 multiplies; the round keys k_r = seed + r * (0x9E3779B9,
// 0xBB67AE85) mod 2^32 (the Weyl bumps) are computed once on the host, so
// each round xors a kernel-parameter constant.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ uint4 philox10_keys(uint4 c, const PhiloxKeys& k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k.k0[r], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k.k1[r], static_cast<uint32_t>(p0));
  }
  return c;
}

__device__ __forceinline__ float code_byte_f(uint32_t q4, int i) {
  return __fsub_rn(__int_as_float(0x4B400000 + static_cast<int>(static_cast<int8_t>(q4 >> (8 * i)))),
                   12582912.0f);
}

// wv[e] = s * code_byte_f(q4, e), two at a time (for products that are
// multiplied next, not added to).
__device__ __forceinline__ void dequant4(uint32_t q4, float s, float (&wv)[4]) {
  const float2 mg = make_float2(12582912.0f, 12582912.0f), ss = make_float2(s, s);
#pragma unroll
  for (int h = 0; h < 4; h += 2) {
    const float2 b = make_float2(
        __int_as_float(0x4B400000 + static_cast<int>(static_cast<int8_t>(q4 >> (8 * h)))),
        __int_as_float(0x4B400000 + static_cast<int>(static_cast<int8_t>(q4 >> (8 * h + 8)))));
    const float2 p = mul2(ss, sub2(b, mg));
    wv[h] = p.x;
    wv[h + 1] = p.y;
  }
}

// The same update with the row staged by the bulk-copy engine: one CTA per
// row copies the row's codes, gradient and both moments into shared memory
// with four bulk copies on one mbarrier (13 K bytes for AdamW), so every load
// of the row is in flight at once without holding a register, and three such
// CTAs share an SM; the updated float row is parked over the gradient.  Used
// while a row fits twice in the shared memory of one CTA.
__global__ void __launch_bounds__(512, 1) update_sr_staged_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int K,
    UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, PhiloxKeys keys,
    uint32_t step_lo, uint32_t step_hi, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t s_max[16];
  __shared__ __align__(8) uint64_t s_full;
  __shared__ volatile int s_abort;
  // Rows from the last: the gradient rows a preceding GEMM wrote last are the
  // likeliest to be still in L2 (the result does not depend on the order).
  const int n = gridDim.x - 1 - blockIdx.x;
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nch = K >> 2;
  const bool adam = c.kind == QL_ADAMW;
  const uint32_t qbytes = static_cast<uint32_t>(K), fbytes = 4u * static_cast<uint32_t>(K);
  const int64_t row = static_cast<int64_t>(n) * K;
  const uint32_t bar = smem_u32(&s_full);
  griddep_wait();  // the gradient (an earlier kernel's output) is visible from here
  if (t == 0) {
    mbar_init(bar, 1);
    s_abort = 0;
    fence_mbar_init();
    const uint32_t dst = smem_u32(smem);
    mbar_arrive_expect_tx(bar, qbytes + fbytes * (adam ? 3u : 1u));
    bulk_load(dst, wq + row, qbytes, bar);
    bulk_load(dst + qbytes, grad + row, fbytes, bar);
    if (adam) {
      bulk_load(dst + qbytes + fbytes, mom1 + row, fbytes, bar);
      bulk_load(dst + qbytes + 2 * fbytes, mom2 + row, fbytes, bar);
    }
  }
  const float s = sw[n];
  __syncthreads();  // barrier initialised before anyone waits on it
  const bool ok = mbar_wait(bar, 0, &s_abort);
  const uint32_t* q_s = reinterpret_cast<const uint32_t*>(smem);
  float4* g_s = reinterpret_cast<float4*>(smem + qbytes);  // then the updated row
  const float4* m_s = reinterpret_cast<const float4*>(smem + qbytes + fbytes);
  const float4* v_s = reinterpret_cast<const float4*>(smem + qbytes + 2 * fbytes);
  float4* m_out = reinterpret_cast<float4*>(mom1 + row);
  float4* v_out = reinterpret_cast<float4*>(mom2 + row);
  uint32_t mbits = 0;
  if (ok) {
    for (int ch = t; ch < nch; ch += T) {
      const uint32_t q4 = q_s[ch];
      const float4 g4 = g_s[ch];
      const float gr[4] = {g4.x, g4.y, g4.z, g4.w};
      float w[4];
      if (adam) {
        const float4 m4 = m_s[ch];
        const float4 v4 = v_s[ch];
        float m1[4] = {m4.x, m4.y, m4.z, m4.w};
        float m2[4] = {v4.x, v4.y, v4.z, v4.w};
        float wv[4];
        dequant4(q4, s, wv);
        adamw4(c, wv, gr, m1, m2, w);
        __stcs(m_out + ch, make_float4(m1[0], m1[1], m1[2], m1[3]));
        __stcs(v_out + ch, make_float4(m2[0], m2[1], m2[2], m2[3]));
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = s * code_byte_f(q4, e) - c.lr * gr[e];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) mbits = max(mbits, abs_bits(w[e]));
      g_s[ch] = make_float4(w[0], w[1], w[2], w[3]);
    }
  }
  mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
  if (lane == 0) s_max[warp] = mbits;
  __syncthreads();
  if (s_abort) {
    // Timed out: the copies may still be landing; wait for them (bounded)
    // before the CTA's shared memory is released.
    if (t == 0) {
      atomicOr(status, 1 << QL_ERR_TIMEOUT);
      mbar_wait_drain(bar, 0);
    }
    return;
  }
  mbits = 0;
  for (int k = 0; k < nwarps; ++k) mbits = max(mbits, s_max[k]);
  const float amax = __uint_as_float(mbits);
  const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
  if (t == 0) {
    sw[n] = mbits == 0 ? 0.0f : amax / 127.0f;
    if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
  }
  griddep_launch_dependents();
  // Element e = n*K + k uses word e&3 of Philox(counter = (e>>2 lo, e>>2 hi,
  // step lo, step hi), key = seed); chunk ch of this row is block row/4 + ch.
  uint32_t* q_out = reinterpret_cast<uint32_t*>(wq + row);
  const uint64_t blk0 = static_cast<uint64_t>(row) >> 2;
  for (int ch = t; ch < nch; ch += T) {
    const uint64_t blk = blk0 + static_cast<uint64_t>(ch);
    const uint4 rn = philox10_keys(
        make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), step_lo, step_hi),
        keys);
    const float4 w = g_s[ch];
    uint32_t out = 0;
    if (mbits != 0)
      out = sr_codes4(w, inv, rn);
    __stcs(q_out + ch, out);
  }
}

// The row-wise weight-norm update with the row's codes and gradient staged
// in shared memory by two bulk copies, so the gradient is read from HBM once
// although both the direction-gradient reduction and the update use it.
// With MS (AdamW rows that fit three times in an SM's shared memory at 13
// bytes per element, K up to ~5.6K) the two moments are staged by two more
// bulk copies on the same barrier, so every load of the row is in flight at
// once and the elementwise step reads shared memory only (up to 384
// threads, three or more CTAs per SM; with two, as at K = 8192, an SM's
// loads stall while both rows compute, which measured slower than streaming
// the moments).  Otherwise the moments stream through registers in the
// elementwise step (coalesced 16-byte loads issued U chunks ahead), which
// keeps a row at 5 bytes of shared memory per element, so several rows share
// an SM: U = 1 with four CTAs of up to 64 registers while four rows fit an
// SM (K up to ~10.6K), U = 4 with three CTAs of 80 registers for longer
// rows, where shared memory leaves fewer CTAs to hide the loads (512-thread
// CTAs with U = 1 measured slower there).  Only the dg reduction
// keeps 16-element groups: the first L threads (L a power of two <= 256) are
// the virtual lanes of the pinned 256-lane order,
// lane l adding groups l, l+L, ... (L = 256, or each group has its own lane).
// ||q||^2 (an integer sum), the elementwise step, the row max and the
// stochastic rounding are free of order and run on all threads over
// 4-element chunks as in update_sr_staged_kernel (consecutive threads touch
// consecutive 16-byte pieces).  Per-element arithmetic and random words are
// the same IEEE operations as the oracle's, so the results are the same bits.
template <bool MS, int U>
__global__ void __launch_bounds__(MS ? 384 : 256, MS ? 3 : (U == 1 ? 4 : 3)) update_sr_wn_staged_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int K,
    UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, PhiloxKeys keys,
    uint32_t step_lo, uint32_t step_hi, float* __restrict__ gmag, float* __restrict__ g_m,
    float* __restrict__ g_v, int L, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_red[256];
  __shared__ uint32_t s_amax[16];  // row maximum (bits) per warp (s_red may still be read)
  __shared__ float s_qhat[256];  // q / ||q|| for every byte value q = -128 .. 127
  __shared__ float s_dgq[256];   // dg * (q / ||q||), the same table times dg
  __shared__ int s_ired[16];
  __shared__ float s_dg;
  __shared__ __align__(8) uint64_t s_full;  // codes + gradient
  __shared__ volatile int s_abort;
  const int n = gridDim.x - 1 - blockIdx.x;  // rows from the last, as the staged kernel
  const int t = threadIdx.x;
  const int T = blockDim.x;  // multiple of 32, L .. 256 (.. 384 with MS)
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int ngroups = K >> 4, nch = K >> 2;
  const int64_t row = static_cast<int64_t>(n) * K;
  const bool adam = c.kind == QL_ADAMW;
  const uint32_t qbytes = static_cast<uint32_t>(K), fbytes = 4u * static_cast<uint32_t>(K);
  // The codes and the gradient are staged (the reductions need them whole),
  // with MS the moments too.
  const uint32_t bar = smem_u32(&s_full);
  griddep_wait();  // the gradient (an earlier kernel's output) is visible from here
  if (t == 0) {
    mbar_init(bar, 1);
    s_abort = 0;
    fence_mbar_init();
    const uint32_t dst = smem_u32(smem);
    mbar_arrive_expect_tx(bar, qbytes + fbytes * (MS ? 3u : 1u));
    bulk_load(dst, wq + row, qbytes, bar);
    bulk_load(dst + qbytes, grad + row, fbytes, bar);
    if (MS) {
      bulk_load(dst + qbytes + fbytes, mom1 + row, fbytes, bar);
      bulk_load(dst + qbytes + 2 * fbytes, mom2 + row, fbytes, bar);
    }
  }
  const float s = sw[n];
  const float gmag_n = gmag[n];  // read before thread 0 overwrites it
  __syncthreads();
  mbar_wait(bar, 0, &s_abort);
  __syncthreads();
  if (s_abort) {  // uniform: every thread reads the flag after the barrier
    if (t == 0) {  // copies may still be landing: wait for them (bounded)
      atomicOr(status, 1 << QL_ERR_TIMEOUT);
      mbar_wait_drain(bar, 0);
    }
    return;
  }
  const uint32_t* q_s = reinterpret_cast<const uint32_t*>(smem);
  float4* g_s = reinterpret_cast<float4*>(smem + qbytes);  // then the updated direction

  // ||q||^2 as an exact integer sum (<= 127^2 * 32768 < 2^31), four codes
  // a dot-product instruction.
  int ss = 0;
  for (int ch = t; ch < nch; ch += T) {
    const int q4 = static_cast<int>(q_s[ch]);
    ss = __dp4a(q4, q4, ss);
  }
  ss = warp_sum_i(ss);
  if (lane == 0) s_ired[warp] = ss;
  __syncthreads();
  ss = 0;
  for (int k = 0; k < nwarps; ++k) ss += s_ired[k];
  if (ss == 0) {  // a zero direction cannot be normalized: reject the row (uniform)
    if (t == 0) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
    return;
  }
  const float nq = static_cast<float>(sqrt(static_cast<double>(ss)));
  // A code is one byte, so q / ||q|| is a 256-entry table: the same IEEE
  // quotients, computed once per row instead of twice per element.
  for (int cidx = t; cidx < 256; cidx += T) s_qhat[cidx] = static_cast<float>(cidx - 128) / nq;
  __syncthreads();
  // dg in the fixed order: virtual lane t < L adds its groups' products in
  // increasing k; lanes >= L hold +0.
  float p = 0.0f;
  if (t < L) {
    const uint4* q16 = reinterpret_cast<const uint4*>(smem);
    const float* gf = reinterpret_cast<const float*>(smem + qbytes);
    for (int j = t; j < ngroups; j += L) {
      const uint4 q4 = q16[j];
      float gr[16];
      load16f(gf + 16 * j, gr);
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        // products two at a time, added one at a time in increasing k
        const float2 pr = mul2(make_float2(gr[e], gr[e + 1]),
                               make_float2(s_qhat[code_at(q4, e) + 128],
                                           s_qhat[code_at(q4, e + 1) + 128]));
        p = __fadd_rn(p, pr.x);
        p = __fadd_rn(p, pr.y);
      }
    }
  }
  // The butterfly p += p[lane ^ off], off = 128 .. 1, over the 256 virtual
  // lanes.  Levels with off >= L add a partner that holds +0 (once is the
  // same as repeatedly).  The levels 32 <= off < L cross warps: every lane's
  // column of values goes through shared memory once and each thread repeats
  // the levels for all L/32 warps of its column (own + partner, the same
  // additions the partners make), keeping its own warp's result.  The levels
  // below 32 are shuffles.
  if (L < 256) p = p + 0.0f;
  if (L > 32) {
    if (t < L) s_red[t] = p;
    __syncthreads();
    if (t < L) {
      const int W = L >> 5;
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = u < W ? s_red[u * 32 + lane] : 0.0f;
#pragma unroll
      for (int k = 4; k >= 1; k >>= 1) {
        if (k < W) {
          float nv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) nv[u] = v[u] + v[u ^ k];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = nv[u];
        }
      }
      float mine = v[0];
#pragma unroll
      for (int u = 1; u < 8; ++u) mine = warp == u ? v[u] : mine;
      p = mine;
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1)
    if (off < L) p = p + __shfl_xor_sync(0xFFFFFFFFu, p, off);
  // Every lane < L holds the same sum; lanes >= L (T > L) take it from lane 0.
  float dg = p;
  if (L < T) {
    if (t == 0) s_dg = p;
    __syncthreads();
    dg = s_dg;
  }
  const float coef = gmag_n / (s * nq);
  // dg * qhat for every code value, once per row instead of once per element
  for (int cidx = t; cidx < 256; cidx += T) s_dgq[cidx] = __fmul_rn(dg, s_qhat[cidx]);
  __syncthreads();

  // Optimizer step of every element; moments written back as they are done,
  // the updated direction parked over the gradient.
  float4* m_out = reinterpret_cast<float4*>(mom1 + row);
  float4* v_out = reinterpret_cast<float4*>(mom2 + row);
  uint32_t mbits = 0;  // max |w'| as float bits (NaN above inf)
  auto update_chunk = [&](int ch, float (&m1)[4], float (&m2)[4]) {
    const uint32_t q4 = q_s[ch];
    const float4 g4 = g_s[ch];
    const float gr[4] = {g4.x, g4.y, g4.z, g4.w};
    float w[4], gg[4], wv[4], dd[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dd[e] = __fsub_rn(gr[e], s_dgq[static_cast<int>(static_cast<int8_t>(q4 >> (8 * e))) + 128]);
    }
    // coef * (g - dg * qhat) and s * q, two at a time (both are multiplied next)
    const float2 cc = make_float2(coef, coef);
    const float2 g01 = mul2(cc, make_float2(dd[0], dd[1])), g23 = mul2(cc, make_float2(dd[2], dd[3]));
    gg[0] = g01.x; gg[1] = g01.y; gg[2] = g23.x; gg[3] = g23.y;
    if (adam) {
      dequant4(q4, s, wv);
      adamw4(c, wv, gg, m1, m2, w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = __fsub_rn(__fmul_rn(s, code_byte_f(q4, e)), __fmul_rn(c.lr, gg[e]));
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) mbits = max(mbits, abs_bits(w[e]));
    if (adam) {
      __stcs(m_out + ch, make_float4(m1[0], m1[1], m1[2], m1[3]));
      __stcs(v_out + ch, make_float4(m2[0], m2[1], m2[2], m2[3]));
    }
    g_s[ch] = make_float4(w[0], w[1], w[2], w[3]);
  };
  if (MS) {
    const float4* m_s = reinterpret_cast<const float4*>(smem + qbytes + fbytes);
    const float4* v_s = reinterpret_cast<const float4*>(smem + qbytes + 2 * fbytes);
    for (int ch = t; ch < nch; ch += T) {
      const float4 m4 = m_s[ch], v4 = v_s[ch];
      float m1[4] = {m4.x, m4.y, m4.z, m4.w};
      float m2[4] = {v4.x, v4.y, v4.z, v4.w};
      update_chunk(ch, m1, m2);
    }
  } else {
    // U chunks per pass, their moment loads issued together.
    for (int ch0 = t; ch0 < nch; ch0 += U * T) {
      float4 ma[U], va[U];
      if (adam) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int ch = ch0 + u * T;
          if (ch < nch) {
            ma[u] = __ldcs(m_out + ch);
            va[u] = __ldcs(v_out + ch);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int ch = ch0 + u * T;
        if (ch >= nch) break;
        float m1[4], m2[4];
        if (adam) {
          m1[0] = ma[u].x; m1[1] = ma[u].y; m1[2] = ma[u].z; m1[3] = ma[u].w;
          m2[0] = va[u].x; m2[1] = va[u].y; m2[2] = va[u].z; m2[3] = va[u].w;
        }
        update_chunk(ch, m1, m2);
      }
    }
  }
  if (t == 0) {
    float gm = gmag_n;
    if (adam) {
      float a1 = g_m[n], a2 = g_v[n];
      gm = adamw(c, gm, dg, a1, a2);
      g_m[n] = a1;
      g_v[n] = a2;
    } else {
      gm = gm - c.lr * dg;
    }
    gmag[n] = gm;
  }

  // Row max (also the barrier before the scale is overwritten).
  mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
  if (lane == 0) s_amax[warp] = mbits;
  __syncthreads();
  mbits = 0;
  for (int k = 0; k < nwarps; ++k) mbits = max(mbits, s_amax[k]);
  const float amax = __uint_as_float(mbits);
  const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
  if (t == 0) {
    sw[n] = mbits == 0 ? 0.0f : amax / 127.0f;
    if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
  }
  griddep_launch_dependents();
  // Element e = n*K + k uses word e&3 of Philox(counter = (e>>2 lo, e>>2 hi,
  // step lo, step hi), key = seed); chunk ch of this row is block row/4 + ch.
  uint32_t* q_out = reinterpret_cast<uint32_t*>(wq + row);
  const uint64_t blk0 = static_cast<uint64_t>(row) >> 2;
  for (int ch = t; ch < nch; ch += T) {
    const uint64_t blk = blk0 + static_cast<uint64_t>(ch);
    const uint4 rn = philox10_keys(
        make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), step_lo, step_hi),
        keys);
    const float4 w = g_s[ch];
    uint32_t out = 0;
    if (mbits != 0)
      out = sr_codes4(w, inv, rn);
    __stcs(q_out + ch, out);
  }
}

// Rows too long to stage whole (more than ~8.8K elements with AdamW): one
// persistent CTA per SM walks its rows N-1-i for i = blockIdx.x, + gridDim.x, ... while
// a producer warp streams every row's codes, gradient and moments through a
// ring of 2048-element pieces by bulk copies, continuing into the next row
// without a break, so HBM stays busy while the consumers finish a row (its
// row max and stochastic rounding).  16 consumer warps apply the optimizer
// step to each piece as it lands (4-element chunks dealt round-robin, moments
// stored straight back), park the updated row in shared memory (4 K bytes)
// and then, after the row max, draw the Philox words and write the codes.
// Per-element arithmetic and random words are those of the other kernels, so
// the results are the same bits.
constexpr int kRingPiece = 2048;                    // elements per piece (multiple of 16)
constexpr int kRingConsumers = 512;                 // 16 consumer warps
constexpr int kRingThreads = kRingConsumers + 32;   // + the producer warp
constexpr int kRingStagesMax = 4;

// Named barrier 1 over the consumer warps only, OR-reducing a flag: every
// consumer gets the same answer, so they leave a loop together.
__device__ __forceinline__ bool consumers_sync_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(flag ? 1u : 0u), "r"(kRingConsumers)
      : "memory");
  return r != 0;
}

template <bool ADAM>
__global__ void __launch_bounds__(kRingThreads, 1) update_sr_ring_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int64_t N,
    int K, UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, PhiloxKeys keys,
    uint32_t step_lo, uint32_t step_hi, int stages, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int EB = ADAM ? 13 : 5;                                // bytes staged per element
  constexpr uint32_t SB = static_cast<uint32_t>(kRingPiece) * EB;  // bytes per stage
  float4* parked = reinterpret_cast<float4*>(smem + stages * SB);  // the updated row, 4 K bytes
  __shared__ uint32_t s_max[kRingConsumers / 32];
  __shared__ __align__(8) uint64_t s_full[kRingStagesMax], s_empty[kRingStagesMax];
  __shared__ volatile int s_abort;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int npieces = (K + kRingPiece - 1) / kRingPiece;
  if (t == 0) {
    for (int st = 0; st < stages; ++st) {
      mbar_init(smem_u32(&s_full[st]), 1);
      mbar_init(smem_u32(&s_empty[st]), kRingConsumers / 32);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the gradient (an earlier kernel's output) is visible from here
  if (warp == kRingConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, issued_phase = 0;
      bool ok = true;
      int k = 0;
      for (int64_t i = blockIdx.x; i < N && ok; i += gridDim.x) {
        const int64_t n = N - 1 - i;  // rows from the last (see the consumers)
        const int64_t row = n * K;
        for (int p = 0; p < npieces; ++p, ++k) {
          const int st = k % stages;
          const uint32_t ph = static_cast<uint32_t>(k / stages) & 1u;
          if (k >= stages && !mbar_wait(smem_u32(&s_empty[st]), ph ^ 1u, &s_abort)) {
            ok = false;
            break;
          }
          const int e0 = p * kRingPiece;
          const uint32_t ne = static_cast<uint32_t>(min(kRingPiece, K - e0));
          const uint32_t dst = smem_u32(smem + st * SB);
          const uint32_t bar = smem_u32(&s_full[st]);
          mbar_arrive_expect_tx(bar, ne * EB);
          bulk_load(dst, wq + row + e0, ne, bar);
          bulk_load(dst + kRingPiece, grad + row + e0, 4 * ne, bar);
          if (ADAM) {
            bulk_load(dst + 5 * kRingPiece, mom1 + row + e0, 4 * ne, bar);
            bulk_load(dst + 9 * kRingPiece, mom2 + row + e0, 4 * ne, bar);
          }
          issued |= 1u << st;
          issued_phase = (issued_phase & ~(1u << st)) | (ph << st);
        }
      }
      // Every copy issued must land before the CTA may exit.
      for (int st = 0; st < stages; ++st)
        if (issued & (1u << st)) mbar_wait_drain(smem_u32(&s_full[st]), (issued_phase >> st) & 1u);
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  constexpr int T = kRingConsumers;
  const int nch_row = K >> 2;
  int k = 0;
  for (int64_t i = blockIdx.x; i < N; i += gridDim.x) {
    // Rows from the last: the gradient rows a preceding GEMM wrote last are
    // the likeliest to be still in L2 (the result does not depend on the order).
    const int64_t n = N - 1 - i;
    const int64_t row = n * K;
    const float s = sw[n];
    float4* m_out = reinterpret_cast<float4*>(mom1 + row);
    float4* v_out = reinterpret_cast<float4*>(mom2 + row);
    uint32_t mbits = 0;
    bool ok = true;
    for (int p = 0; p < npieces; ++p, ++k) {
      const int st = k % stages;
      const uint32_t ph = static_cast<uint32_t>(k / stages) & 1u;
      if (!mbar_wait(smem_u32(&s_full[st]), ph, &s_abort)) {
        ok = false;
        break;
      }
      const uint8_t* src = smem + st * SB;
      const uint32_t* q_s = reinterpret_cast<const uint32_t*>(src);
      const float4* g_s = reinterpret_cast<const float4*>(src + kRingPiece);
      const float4* m_s = reinterpret_cast<const float4*>(src + 5 * kRingPiece);
      const float4* v_s = reinterpret_cast<const float4*>(src + 9 * kRingPiece);
      const int c0 = (p * kRingPiece) >> 2;
      const int nch = min(kRingPiece, K - p * kRingPiece) >> 2;
      for (int ch = t; ch < nch; ch += T) {
        const uint32_t q4 = q_s[ch];
        const float4 g4 = g_s[ch];
        const float gr[4] = {g4.x, g4.y, g4.z, g4.w};
        float w[4];
        if (ADAM) {
          const float4 m4 = m_s[ch];
          const float4 v4 = v_s[ch];
          float m1[4] = {m4.x, m4.y, m4.z, m4.w};
          float m2[4] = {v4.x, v4.y, v4.z, v4.w};
          float wv[4];
          dequant4(q4, s, wv);
          adamw4(c, wv, gr, m1, m2, w);
          __stcs(m_out + c0 + ch, make_float4(m1[0], m1[1], m1[2], m1[3]));
          __stcs(v_out + c0 + ch, make_float4(m2[0], m2[1], m2[2], m2[3]));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = s * code_byte_f(q4, e) - c.lr * gr[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) mbits = max(mbits, abs_bits(w[e]));
        parked[c0 + ch] = make_float4(w[0], w[1], w[2], w[3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_empty[st]));
    }
    mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
    if (lane == 0) s_max[warp] = mbits;
    // Row max complete and the parked row written; leave together on abort.
    if (consumers_sync_or(!ok || s_abort)) break;
    mbits = 0;
#pragma unroll
    for (int w8 = 0; w8 < T / 32; ++w8) mbits = max(mbits, s_max[w8]);
    const float amax = __uint_as_float(mbits);
    const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
    if (t == 0) {
      sw[n] = mbits == 0 ? 0.0f : amax / 127.0f;
      if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
    }
    // Element e = n*K + k uses word e&3 of Philox(counter = (e>>2 lo, e>>2 hi,
    // step lo, step hi), key = seed); chunk ch of this row is block row/4 + ch.
    uint32_t* q_out = reinterpret_cast<uint32_t*>(wq + row);
    const uint64_t blk0 = static_cast<uint64_t>(row) >> 2;
    for (int ch = t; ch < nch_row; ch += T) {
      const uint64_t blk = blk0 + static_cast<uint64_t>(ch);
      const uint4 rn = philox10_keys(
          make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), step_lo, step_hi),
          keys);
      const float4 w = parked[ch];
      uint32_t out = 0;
      if (mbits != 0)
        out = sr_codes4(w, inv, rn);
      __stcs(q_out + ch, out);
    }
    // s_max and the parked row are rewritten by the next row.
    if (consumers_sync_or(s_abort)) break;
  }
  griddep_launch_dependents();
  if (t == 0 && s_abort) atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

// The Muon step of an int8 weight from its orthogonalized update O (bf16
// [N, K]): w = s*q; w' = (w*a) - st*O, one rounding per operation; then the
// row max and the Philox-keyed stochastic rounding of the other updates.  One
// CTA per row stages the row's codes and O by two bulk copies on one mbarrier
// (3 bytes per element, so every load of the row is in flight at once),
// 4-element chunks dealt round-robin, the updated row parked in shared
// memory (4 K bytes).
__global__ void __launch_bounds__(512) update_sr_dir_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const __nv_bfloat16* __restrict__ O, int K,
    float a, float st, PhiloxKeys keys, uint32_t step_lo, uint32_t step_hi,
    int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t s_max[16];
  __shared__ __align__(8) uint64_t s_full;
  __shared__ volatile int s_abort;
  const int n = blockIdx.x, t = threadIdx.x, T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nch = K >> 2;
  const int64_t row = static_cast<int64_t>(n) * K;
  const uint32_t qbytes = static_cast<uint32_t>(K), obytes = 2u * static_cast<uint32_t>(K);
  float4* s_w = reinterpret_cast<float4*>(smem);  // the updated row (4 K bytes)
  const uint32_t bar = smem_u32(&s_full);
  if (t == 0) {
    mbar_init(bar, 1);
    s_abort = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, qbytes + obytes);
    bulk_load(smem_u32(smem) + 4u * K, wq + row, qbytes, bar);
    bulk_load(smem_u32(smem) + 5u * K, O + row, obytes, bar);
  }
  const float s = sw[n];
  __syncthreads();  // barrier initialised before anyone waits on it
  const bool ok = mbar_wait(bar, 0, &s_abort);
  const uint32_t* q_in = reinterpret_cast<const uint32_t*>(smem + 4 * K);
  const uint2* o_in = reinterpret_cast<const uint2*>(smem + 5 * K);
  uint32_t mbits = 0;
  for (int ch = t; ok && ch < nch; ch += T) {
    const uint32_t q4 = q_in[ch];
    const uint2 o2 = o_in[ch];
    const float o[4] = {__uint_as_float(o2.x << 16), __uint_as_float(o2.x & 0xFFFF0000u),
                        __uint_as_float(o2.y << 16), __uint_as_float(o2.y & 0xFFFF0000u)};
    float w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      w[e] = (s * code_byte_f(q4, e)) * a - st * o[e];
      mbits = max(mbits, abs_bits(w[e]));
    }
    s_w[ch] = make_float4(w[0], w[1], w[2], w[3]);
  }
  mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
  if (lane == 0) s_max[warp] = mbits;
  __syncthreads();
  if (s_abort) {
    if (t == 0) {  // timed out: wait (bounded) for the copies before the CTA exits
      atomicOr(status, 1 << QL_ERR_TIMEOUT);
      mbar_wait_drain(bar, 0);
    }
    return;
  }
  mbits = 0;
  for (int k = 0; k < nwarps; ++k) mbits = max(mbits, s_max[k]);
  const float amax = __uint_as_float(mbits);
  const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
  if (t == 0) {
    sw[n] = mbits == 0 ? 0.0f : amax / 127.0f;
    if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
  }
  uint32_t* q_out = reinterpret_cast<uint32_t*>(wq + row);
  const uint64_t blk0 = static_cast<uint64_t>(row) >> 2;
  for (int ch = t; ch < nch; ch += T) {
    const uint64_t blk = blk0 + static_cast<uint64_t>(ch);
    const uint4 rn = philox10_keys(
        make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), step_lo, step_hi),
        keys);
    const float4 w = s_w[ch];
    uint32_t out = 0;
    if (mbits != 0)
      out = sr_codes4(w, inv, rn);
    __stcs(q_out + ch, out);
  }
}


// Chunks of 4 elements per thread (sets the thread count of both kernels).
#ifndef QL_UPDATE_STAGED_CHUNKS
#define QL_UPDATE_STAGED_CHUNKS 4
#endif

}  // namespace

cudaError_t launch_update_sr(int8_t* wq, float* sw, const float* grad, int64_t N, int64_t K,
                             const UpdateConsts& c, float* m, float* v, uint64_t seed,
                             uint64_t step, float* g, float* g_m, float* g_v, int32_t* status,
                             cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  const int ngroups = static_cast<int>(K / 16);
  int T = 32;
  while (T < ngroups && T < 256) T <<= 1;
  const uint32_t sl = static_cast<uint32_t>(seed), sh = static_cast<uint32_t>(seed >> 32);
  const uint32_t tl = static_cast<uint32_t>(step), th = static_cast<uint32_t>(step >> 32);
  const int k = static_cast<int>(K);
  const unsigned grid = static_cast<unsigned>(N);
  if (g != nullptr) {
    // Weight norm: the row's codes and gradient staged (5 bytes per
    // element, every K <= 32768 fits), and with AdamW the moments too when
    // three such rows fit an SM (13 bytes per element, K up to ~5.6K); at
    // most 256 threads (384 with the moments staged), of which the first L
    // are the pinned reduction's virtual lanes.
    const int nch = static_cast<int>(K / 4);
    const int64_t full_bytes = 13 * K;
    // (an SM has 1 KB more shared memory than one CTA may take; 5 KB covers
    // the kernel's static arrays and the per-CTA reserve)
    const bool ms = c.kind == QL_ADAMW &&
                    3 * (full_bytes + 5120) <= device_info().smem_optin + 1024;
    // Streamed moments: one chunk ahead while four rows fit an SM, four
    // chunks ahead otherwise.
    const bool u1 = 4 * (5 * K + 5120) <= device_info().smem_optin + 1024;
    const int variant = ms ? 0 : (u1 ? 1 : 2);
    const int64_t row_bytes = ms ? full_bytes : 5 * K;
    static bool wn_set[3][64] = {{false}};
    int dev = 0;
    cudaGetDevice(&dev);
    auto kern = variant == 0 ? update_sr_wn_staged_kernel<true, 1>
                : variant == 1 ? update_sr_wn_staged_kernel<false, 1>
                               : update_sr_wn_staged_kernel<false, 4>;
    if (dev < 64 && !__atomic_load_n(&wn_set[variant][dev], __ATOMIC_ACQUIRE)) {
      cudaFuncAttributes fa{};
      e = cudaFuncGetAttributes(&fa, kern);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 device_info().smem_optin - static_cast<int>(fa.sharedSizeBytes));
      if (e != cudaSuccess) {
        (void)cudaGetLastError();  // returned here; not left for a later check
        return e;
      }
      __atomic_store_n(&wn_set[variant][dev], true, __ATOMIC_RELEASE);
    }
    PhiloxKeys keys;
    for (int r = 0; r < 10; ++r) {
      keys.k0[r] = sl + static_cast<uint32_t>(r) * 0x9E3779B9u;
      keys.k1[r] = sh + static_cast<uint32_t>(r) * 0xBB67AE85u;
    }
    const int tmax = ms ? 384 : 256;
    const int tr = std::max(T, std::min(tmax, std::max(32, (nch / QL_UPDATE_STAGED_CHUNKS + 31) / 32 * 32)));
    e = launch_pdl(kern, dim3(grid), dim3(tr), static_cast<size_t>(row_bytes), s, wq, sw, grad, k,
                   c, m, v, keys, tl, th, g, g_m, g_v, T, status);
    count_launches(1);
    return e == cudaSuccess ? cudaGetLastError() : e;
  } else {
    const int nch = static_cast<int>(K / 4);
    PhiloxKeys keys;
    for (int r = 0; r < 10; ++r) {
      keys.k0[r] = sl + static_cast<uint32_t>(r) * 0x9E3779B9u;
      keys.k1[r] = sh + static_cast<uint32_t>(r) * 0xBB67AE85u;
    }
    const int64_t row_bytes = K * (c.kind == QL_ADAMW ? 13 : 5);
    const int64_t budget = device_info().smem_optin - 1024;
    if (2 * (row_bytes + 1024) <= budget) {
      const int tr = std::min(512, std::max(32, (nch / QL_UPDATE_STAGED_CHUNKS + 31) / 32 * 32));
      static bool staged_set[64] = {false};
      int dev = 0;
      cudaGetDevice(&dev);
      if (dev < 64 && !__atomic_load_n(&staged_set[dev], __ATOMIC_ACQUIRE)) {
        cudaFuncSetAttribute(update_sr_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(budget));
        __atomic_store_n(&staged_set[dev], true, __ATOMIC_RELEASE);
      }
      e = launch_pdl(update_sr_staged_kernel, dim3(grid), dim3(tr), static_cast<size_t>(row_bytes),
                     s, wq, sw, grad, k, c, m, v, keys, tl, th, status);
      count_launches(1);
      return e == cudaSuccess ? cudaGetLastError() : e;
    }
    // Longer rows: the piece ring, with as many stages as fit beside the
    // parked row (4 K bytes).
    {
      const int64_t stage_bytes = static_cast<int64_t>(kRingPiece) * (c.kind == QL_ADAMW ? 13 : 5);
      const int64_t ring_budget = device_info().smem_optin - 1024 - 4 * K;
      const int stages = static_cast<int>(std::min<int64_t>(kRingStagesMax, ring_budget / stage_bytes));
      if (stages >= 2) {
        const size_t smem = static_cast<size_t>(stages * stage_bytes + 4 * K);
        static bool ring_set[64] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 64 && !__atomic_load_n(&ring_set[dev], __ATOMIC_ACQUIRE)) {
          cudaFuncSetAttribute(update_sr_ring_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               device_info().smem_optin - 1024);
          cudaFuncSetAttribute(update_sr_ring_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               device_info().smem_optin - 1024);
          __atomic_store_n(&ring_set[dev], true, __ATOMIC_RELEASE);
        }
        const unsigned rgrid = static_cast<unsigned>(std::min<int64_t>(N, device_info().sms));
        if (c.kind == QL_ADAMW)
          e = launch_pdl(update_sr_ring_kernel<true>, dim3(rgrid), dim3(kRingThreads), smem, s, wq,
                         sw, grad, N, k, c, m, v, keys, tl, th, stages, status);
        else
          e = launch_pdl(update_sr_ring_kernel<false>, dim3(rgrid), dim3(kRingThreads), smem, s, wq,
                         sw, grad, N, k, c, m, v, keys, tl, th, stages, status);
        count_launches(1);
        return e == cudaSuccess ? cudaGetLastError() : e;
      }
    }
    return cudaErrorInvalidConfiguration;  // unreachable for K <= 32768
  }
}

cudaError_t launch_update_dir(int8_t* wq, float* sw, const void* O, int64_t N, int64_t K, float a,
                              float st, uint64_t seed, uint64_t step, int32_t* status,
                              cudaStream_t s) {
  PhiloxKeys keys;
  const uint32_t sl = static_cast<uint32_t>(seed), sh = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    keys.k0[r] = sl + static_cast<uint32_t>(r) * 0x9E3779B9u;
    keys.k1[r] = sh + static_cast<uint32_t>(r) * 0xBB67AE85u;
  }
  static bool dir_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !__atomic_load_n(&dir_set[dev], __ATOMIC_ACQUIRE)) {
    cudaFuncSetAttribute(update_sr_dir_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         7 * 32768);
    __atomic_store_n(&dir_set[dev], true, __ATOMIC_RELEASE);
  }
  const int nch = static_cast<int>(K / 4);
  const int tr = std::min(512, std::max(32, (nch / 4 + 31) / 32 * 32));
  // the updated row (4 bytes per element), then the staged codes (1) and O (2)
  update_sr_dir_kernel<<<static_cast<unsigned>(N), tr, static_cast<size_t>(7) * K, s>>>(
      wq, sw, reinterpret_cast<const __nv_bfloat16*>(O), static_cast<int>(K), a, st, keys,
      static_cast<uint32_t>(step), static_cast<uint32_t>(step >> 32), status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ql
