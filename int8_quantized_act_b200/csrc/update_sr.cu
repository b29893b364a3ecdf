// update_sr.cu - fused optimizer step + stochastic requantization of int8
// weight rows (mini_trainer "docs/quantized-training.md": the paragraph after
// the feature table - updates requantize the represented weights
// stochastically in CUDA row kernels, with no floating master weight; feature
// table rows "Optimizers" and "Row-wise weight normalization").
//
// One CTA owns one weight row and reads it from HBM once: codes, gradient
// and moments in, new moments out, while the updated float row waits in
// shared memory for the row max; the new scale follows from a CTA max
// reduction; then every 4-element chunk draws one Philox4x32-10 block and
// writes 4 stochastically rounded codes.  Rows up to ~8K elements are staged
// whole by the bulk-copy engine (update_sr_staged_kernel); longer rows are
// loaded through registers (update_sr_rows_kernel).  The row-wise weight-norm
// variant stages its row the same way (update_sr_wn_staged_kernel; beyond
// shared memory, update_sr_kernel) and keeps 16-element groups only for the
// pinned order of its direction-gradient reduction.  Bytes per element:
// AdamW 22 (1+4+4+4 in, 1+4+4 out), SGD 6.
#include <cuda_runtime.h>

#include <algorithm>

#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of two
// 32x32->64 multiplies, key bumped by the Weyl constants between rounds.
__device__ __forceinline__ uint4 philox10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;  // one 32x32->64 multiply
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k0, static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k1, static_cast<uint32_t>(p0));
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

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

// floor(v) + 1 with probability frac(v), decided by u24 < frac * 2^24;
// clamped to [-127, 127].  Returns rne_bits of the (integer-valued) result, so
// its low byte is the int8 code (exact: adding 1.5*2^23 to an integer-valued
// float below 2^22 in magnitude is exact).
__device__ __forceinline__ uint32_t sr_code_bits(float val, uint32_t u24) {
  const float f = floorf(val);
  const float frac = val - f;
  float r = (__uint2float_rn(u24) < frac * 16777216.0f) ? f + 1.0f : f;
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return rne_bits(r);
}

// Stochastic codes of 16 consecutive elements starting at element e0
// (a multiple of 16): four Philox blocks, word e & 3 of block e >> 2.
__device__ __forceinline__ uint4 sr_group(const float (&w)[16], float inv, bool zero_row,
                                          uint64_t e0, uint32_t sl, uint32_t sh, uint32_t tl,
                                          uint32_t th) {
  uint32_t b[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint64_t blk = (e0 >> 2) + k;
    const uint4 r = philox10(make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32),
                                        tl, th),
                             sl, sh);
    const uint32_t words[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      b[4 * k + e] = zero_row ? 0u : sr_code_bits(w[4 * k + e] * inv, words[e] >> 8);
  }
  return make_uint4(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]),
                    pack_codes(b[8], b[9], b[10], b[11]), pack_codes(b[12], b[13], b[14], b[15]));
}

__device__ __forceinline__ void load16f(const float* p, float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 a = reinterpret_cast<const float4*>(p)[i];
    v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
  }
}

__device__ __forceinline__ void store16f(float* p, const float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

__device__ __forceinline__ int code_at(const uint4& q, int i) {
  const uint32_t w = (&q.x)[i >> 2];
  return static_cast<int>(static_cast<int8_t>((w >> (8 * (i & 3))) & 0xFFu));
}

// The int8 code as a float without the conversion unit: 1.5*2^23 + q is
// exact in float32 and its bit pattern is that of 1.5*2^23 plus q.
__device__ __forceinline__ float code_f(const uint4& q, int i) {
  return __fsub_rn(__int_as_float(0x4B400000 + code_at(q, i)), 12582912.0f);
}

template <int GPT, bool WN>
__global__ void __launch_bounds__(256) update_sr_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int K,
    UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, uint32_t seed_lo,
    uint32_t seed_hi, uint32_t step_lo, uint32_t step_hi, float* __restrict__ gmag,
    float* __restrict__ g_m, float* __restrict__ g_v, int32_t* __restrict__ status) {
  __shared__ float s_red[256];
  __shared__ int s_ired[8];
  const int n = blockIdx.x;
  const int t = threadIdx.x;
  const int T = blockDim.x;  // power of two, <= 256
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int ngroups = K >> 4;
  const int64_t row = static_cast<int64_t>(n) * K;
  const bool adam = c.kind == QL_ADAMW;

  const float s = sw[n];
  // The magnitude is read before thread 0 may overwrite it (after the update).
  const float gmag_n = WN ? gmag[n] : 0.0f;
  uint4 qv[GPT];
  float w[GPT][16];
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int j = t + T * i;
    qv[i] = j < ngroups ? *reinterpret_cast<const uint4*>(wq + row + 16 * j) : make_uint4(0, 0, 0, 0);
  }

  float dg = 0.0f, nq = 0.0f, coef = 0.0f;
  if constexpr (WN) {
    // ||q||^2 as an exact integer sum (<= 127^2 * 32768 < 2^31).
    int ss = 0;
#pragma unroll
    for (int i = 0; i < GPT; ++i)
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int qc = code_at(qv[i], e);
        ss += qc * qc;
      }
    ss = warp_sum_i(ss);
    if (lane == 0) s_ired[warp] = ss;
    __syncthreads();
    ss = 0;
    for (int k = 0; k < nwarps; ++k) ss += s_ired[k];
    if (ss == 0) {  // a zero direction cannot be normalized: reject the row
      if (t == 0) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
      return;
    }
    nq = static_cast<float>(sqrt(static_cast<double>(ss)));
    // dg in the fixed order: thread t is lane t of 256 virtual lanes, adding
    // its groups' products in increasing k; lanes >= T hold +0.
    float p = 0.0f;
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
      const int j = t + T * i;
      if (j < ngroups) {
        float gr[16];
        load16f(grad + row + 16 * j, gr);
#pragma unroll
        for (int e = 0; e < 16; ++e) p = p + gr[e] * (code_f(qv[i], e) / nq);
      }
    }
    for (int off = 128; off >= 1; off >>= 1) {
      if (off >= T) {
        p = p + 0.0f;
      } else if (off >= 32) {
        s_red[t] = p;
        __syncthreads();
        const float o = s_red[t ^ off];
        __syncthreads();
        p = p + o;
      } else {
        p = p + __shfl_xor_sync(0xFFFFFFFFu, p, off);
      }
    }
    dg = p;
    coef = gmag_n / (s * nq);
  }

  // Optimizer step of every element; moments written back immediately.
  float amax = 0.0f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int j = t + T * i;
    if (j < ngroups) {
      const int64_t off = row + 16 * j;
      float gr[16], m1[16], m2[16];
      load16f(grad + off, gr);
      if (adam) {
        load16f(mom1 + off, m1);
        load16f(mom2 + off, m2);
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float qf = code_f(qv[i], e);
        float gg = gr[e];
        if constexpr (WN) gg = coef * (gr[e] - dg * (qf / nq));
        const float wv = s * qf;
        w[i][e] = adam ? adamw(c, wv, gg, m1[e], m2[e]) : wv - c.lr * gg;
        bad |= !finite(w[i][e]);
        amax = fmaxf(amax, fabsf(w[i][e]));
      }
      if (adam) {
        store16f(mom1 + off, m1);
        store16f(mom2 + off, m2);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) w[i][e] = 0.0f;
    }
  }
  if constexpr (WN) {
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
  }

  // Row max (also the barrier before the scale is overwritten).
  amax = warp_max(amax);
  bad = warp_or(bad);
  __syncthreads();
  if (lane == 0) {
    s_red[warp] = amax;
    s_ired[warp] = bad;
  }
  __syncthreads();
  amax = 0.0f;
  bad = 0;
  for (int k = 0; k < nwarps; ++k) {
    amax = fmaxf(amax, s_red[k]);
    bad |= s_ired[k];
  }
  const float inv = amax == 0.0f ? 0.0f : 127.0f / amax;
  if (t == 0) {
    sw[n] = amax == 0.0f ? 0.0f : amax / 127.0f;
    if (bad) atomicOr(status, 1 << QL_ERR_NONFINITE);
  }

  // Stochastic requantization: element e = n*K + k uses word e&3 of
  // Philox(counter = (e>>2 lo, e>>2 hi, step lo, step hi), key = seed).
#pragma unroll
  for (int i = 0; i < GPT; ++i) {
    const int j = t + T * i;
    if (j < ngroups)
      *reinterpret_cast<uint4*>(wq + row + 16 * j) =
          sr_group(w[i], inv, amax == 0.0f, static_cast<uint64_t>(row + 16 * j), seed_lo, seed_hi,
                   step_lo, step_hi);
  }
}

// Philox round keys k_r = seed + r * (0x9E3779B9, 0xBB67AE85) mod 2^32,
// computed once on the host so each round xors a kernel-parameter constant.
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

// The plain (not weight-normalized) update.  One CTA per weight row; the row
// is cut into 4-element chunks (one Philox block each) dealt round-robin to
// the threads, so every global access of a warp is one contiguous run.
// Phase 1 streams codes, gradient and moments in, writes the new moments and
// parks the updated float row in shared memory (4 K bytes) while keeping the
// running max of |w'|; phase 2, after the CTA max reduction, draws the Philox
// words and writes the stochastically rounded codes.  Parking the row in
// shared memory instead of registers keeps the register count low, so
// several rows are in flight per SM and their loads overlap the arithmetic.
__global__ void __launch_bounds__(512, 2) update_sr_rows_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int K,
    UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, PhiloxKeys keys,
    uint32_t step_lo, uint32_t step_hi, int32_t* __restrict__ status) {
  extern __shared__ float4 s_row[];
  __shared__ uint32_t s_max[16];
  const int n = blockIdx.x;
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nch = K >> 2;
  const int64_t row = static_cast<int64_t>(n) * K;
  const bool adam = c.kind == QL_ADAMW;
  const float s = sw[n];
  const uint32_t* q_in = reinterpret_cast<const uint32_t*>(wq + row);
  const float4* g_in = reinterpret_cast<const float4*>(grad + row);
  float4* m_io = reinterpret_cast<float4*>(mom1 + row);
  float4* v_io = reinterpret_cast<float4*>(mom2 + row);

  uint32_t mbits = 0;
#pragma unroll 2
  for (int ch = t; ch < nch; ch += T) {
    const uint32_t q4 = __ldcs(q_in + ch);
    const float4 g4 = __ldcs(g_in + ch);
    float gr[4] = {g4.x, g4.y, g4.z, g4.w};
    float w[4];
    if (adam) {
      const float4 m4 = __ldcs(m_io + ch);
      const float4 v4 = __ldcs(v_io + ch);
      float m1[4] = {m4.x, m4.y, m4.z, m4.w};
      float m2[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = adamw(c, s * code_byte_f(q4, e), gr[e], m1[e], m2[e]);
      __stcs(m_io + ch, make_float4(m1[0], m1[1], m1[2], m1[3]));
      __stcs(v_io + ch, make_float4(m2[0], m2[1], m2[2], m2[3]));
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = s * code_byte_f(q4, e) - c.lr * gr[e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) mbits = max(mbits, abs_bits(w[e]));
    s_row[ch] = make_float4(w[0], w[1], w[2], w[3]);
  }
  mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
  if (lane == 0) s_max[warp] = mbits;
  __syncthreads();
  mbits = 0;
  for (int k = 0; k < nwarps; ++k) mbits = max(mbits, s_max[k]);
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
#pragma unroll 2
  for (int ch = t; ch < nch; ch += T) {
    const uint64_t blk = blk0 + static_cast<uint64_t>(ch);
    const uint4 r = philox10_keys(
        make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), step_lo, step_hi),
        keys);
    const float4 w = s_row[ch];
    uint32_t out = 0;
    if (mbits != 0)
      out = pack_codes(sr_code_bits(w.x * inv, r.x >> 8), sr_code_bits(w.y * inv, r.y >> 8),
                       sr_code_bits(w.z * inv, r.z >> 8), sr_code_bits(w.w * inv, r.w >> 8));
    __stcs(q_out + ch, out);
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
  const int n = blockIdx.x;
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int nch = K >> 2;
  const bool adam = c.kind == QL_ADAMW;
  const uint32_t qbytes = static_cast<uint32_t>(K), fbytes = 4u * static_cast<uint32_t>(K);
  const int64_t row = static_cast<int64_t>(n) * K;
  const uint32_t bar = smem_u32(&s_full);
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
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = adamw(c, s * code_byte_f(q4, e), gr[e], m1[e], m2[e]);
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
      out = pack_codes(sr_code_bits(w.x * inv, rn.x >> 8), sr_code_bits(w.y * inv, rn.y >> 8),
                       sr_code_bits(w.z * inv, rn.z >> 8), sr_code_bits(w.w * inv, rn.w >> 8));
    __stcs(q_out + ch, out);
  }
}

// The row-wise weight-norm update with the row staged in shared memory by
// four bulk copies, so the gradient is read from HBM once although both the
// direction-gradient reduction and the update use it; codes and gradient
// land on one barrier, the moments on a second while the reductions run.
// Only the dg reduction keeps 16-element groups: the first L threads (L a
// power of two <= 256) are the virtual lanes of the pinned 256-lane order,
// lane l adding groups l, l+L, ... (L = 256, or each group has its own lane).
// ||q||^2 (an integer sum), the elementwise step, the row max and the
// stochastic rounding are free of order and run on all threads over
// 4-element chunks as in update_sr_staged_kernel (consecutive threads touch
// consecutive 16-byte pieces).  Per-element arithmetic and random words are
// those of update_sr_kernel<GPT, true>, so the results are the same bits.
__global__ void __launch_bounds__(512) update_sr_wn_staged_kernel(
    int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ grad, int K,
    UpdateConsts c, float* __restrict__ mom1, float* __restrict__ mom2, PhiloxKeys keys,
    uint32_t step_lo, uint32_t step_hi, float* __restrict__ gmag, float* __restrict__ g_m,
    float* __restrict__ g_v, int L, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_red[256];
  __shared__ float s_qhat[256];  // q / ||q|| for every byte value q = -128 .. 127
  __shared__ int s_ired[16];
  __shared__ float s_dg;
  __shared__ __align__(8) uint64_t s_full[2];  // codes + gradient; moments
  __shared__ volatile int s_abort;
  const int n = blockIdx.x;
  const int t = threadIdx.x;
  const int T = blockDim.x;  // multiple of 32, L .. 512
  const int warp = t >> 5, lane = t & 31, nwarps = T >> 5;
  const int ngroups = K >> 4, nch = K >> 2;
  const int64_t row = static_cast<int64_t>(n) * K;
  const bool adam = c.kind == QL_ADAMW;
  const uint32_t qbytes = static_cast<uint32_t>(K), fbytes = 4u * static_cast<uint32_t>(K);
  // Two barriers: the reductions need only the codes and the gradient, so
  // they run while the moments are still arriving.
  const uint32_t bar = smem_u32(&s_full[0]), bar_mv = smem_u32(&s_full[1]);
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_mv, 1);
    s_abort = 0;
    fence_mbar_init();
    const uint32_t dst = smem_u32(smem);
    mbar_arrive_expect_tx(bar, qbytes + fbytes);
    bulk_load(dst, wq + row, qbytes, bar);
    bulk_load(dst + qbytes, grad + row, fbytes, bar);
    if (adam) {
      mbar_arrive_expect_tx(bar_mv, 2 * fbytes);
      bulk_load(dst + qbytes + fbytes, mom1 + row, fbytes, bar_mv);
      bulk_load(dst + qbytes + 2 * fbytes, mom2 + row, fbytes, bar_mv);
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
      if (adam) mbar_wait_drain(bar_mv, 0);
    }
    return;
  }
  const uint32_t* q_s = reinterpret_cast<const uint32_t*>(smem);
  float4* g_s = reinterpret_cast<float4*>(smem + qbytes);  // then the updated direction
  const float4* m_s = reinterpret_cast<const float4*>(smem + qbytes + fbytes);
  const float4* v_s = reinterpret_cast<const float4*>(smem + qbytes + 2 * fbytes);

  // ||q||^2 as an exact integer sum (<= 127^2 * 32768 < 2^31).
  int ss = 0;
  for (int ch = t; ch < nch; ch += T) {
    const uint32_t q4 = q_s[ch];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int qc = static_cast<int8_t>(q4 >> (8 * e));
      ss += qc * qc;
    }
  }
  ss = warp_sum_i(ss);
  if (lane == 0) s_ired[warp] = ss;
  __syncthreads();
  ss = 0;
  for (int k = 0; k < nwarps; ++k) ss += s_ired[k];
  if (ss == 0) {  // a zero direction cannot be normalized: reject the row (uniform)
    if (t == 0) {
      atomicOr(status, 1 << QL_ERR_ZERO_ROW);
      if (adam) mbar_wait_drain(bar_mv, 0);  // the moments' copies end first
    }
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
      for (int e = 0; e < 16; ++e) p = p + gr[e] * s_qhat[code_at(q4, e) + 128];
    }
  }
  for (int off = 128; off >= 1; off >>= 1) {
    if (off >= L) {
      p = p + 0.0f;
    } else if (off >= 32) {
      if (t < L) s_red[t] = p;
      __syncthreads();
      const float o = t < L ? s_red[t ^ off] : 0.0f;
      __syncthreads();
      p = p + o;
    } else {
      p = p + __shfl_xor_sync(0xFFFFFFFFu, p, off);
    }
  }
  if (t == 0) s_dg = p;  // every lane < L holds the same sum
  if (adam) mbar_wait(bar_mv, 0, &s_abort);
  __syncthreads();
  if (s_abort) {
    if (t == 0) {
      atomicOr(status, 1 << QL_ERR_TIMEOUT);
      mbar_wait_drain(bar_mv, 0);
    }
    return;
  }
  const float dg = s_dg;
  const float coef = gmag_n / (s * nq);

  // Optimizer step of every element; moments written back as they are done,
  // the updated direction parked over the gradient.
  float4* m_out = reinterpret_cast<float4*>(mom1 + row);
  float4* v_out = reinterpret_cast<float4*>(mom2 + row);
  float amax = 0.0f;
  int bad = 0;
  for (int ch = t; ch < nch; ch += T) {
    const uint32_t q4 = q_s[ch];
    const float4 g4 = g_s[ch];
    const float gr[4] = {g4.x, g4.y, g4.z, g4.w};
    float m1[4], m2[4];
    if (adam) {
      const float4 a = m_s[ch], b = v_s[ch];
      m1[0] = a.x; m1[1] = a.y; m1[2] = a.z; m1[3] = a.w;
      m2[0] = b.x; m2[1] = b.y; m2[2] = b.z; m2[3] = b.w;
    }
    float w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float qhat = s_qhat[static_cast<int>(static_cast<int8_t>(q4 >> (8 * e))) + 128];
      const float gg = coef * (gr[e] - dg * qhat);
      const float wv = s * code_byte_f(q4, e);
      w[e] = adam ? adamw(c, wv, gg, m1[e], m2[e]) : wv - c.lr * gg;
      bad |= !finite(w[e]);
      amax = fmaxf(amax, fabsf(w[e]));
    }
    if (adam) {
      __stcs(m_out + ch, make_float4(m1[0], m1[1], m1[2], m1[3]));
      __stcs(v_out + ch, make_float4(m2[0], m2[1], m2[2], m2[3]));
    }
    g_s[ch] = make_float4(w[0], w[1], w[2], w[3]);
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
  amax = warp_max(amax);
  bad = warp_or(bad);
  if (lane == 0) {
    s_red[warp] = amax;
    s_ired[warp] = bad;
  }
  __syncthreads();
  amax = 0.0f;
  bad = 0;
  for (int k = 0; k < nwarps; ++k) {
    amax = fmaxf(amax, s_red[k]);
    bad |= s_ired[k];
  }
  const float inv = amax == 0.0f ? 0.0f : 127.0f / amax;
  if (t == 0) {
    sw[n] = amax == 0.0f ? 0.0f : amax / 127.0f;
    if (bad) atomicOr(status, 1 << QL_ERR_NONFINITE);
  }
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
    if (amax != 0.0f)
      out = pack_codes(sr_code_bits(w.x * inv, rn.x >> 8), sr_code_bits(w.y * inv, rn.y >> 8),
                       sr_code_bits(w.z * inv, rn.z >> 8), sr_code_bits(w.w * inv, rn.w >> 8));
    __stcs(q_out + ch, out);
  }
}

// Chunks of 4 elements per thread (sets the thread count of both kernels).
#ifndef QL_UPDATE_STAGED_CHUNKS
#define QL_UPDATE_STAGED_CHUNKS 4
#endif
#ifndef QL_UPDATE_CHUNKS_PER_THREAD
#define QL_UPDATE_CHUNKS_PER_THREAD 4
#endif

}  // namespace

cudaError_t launch_update_sr(int8_t* wq, float* sw, const float* grad, int64_t N, int64_t K,
                             const UpdateConsts& c, float* m, float* v, uint64_t seed,
                             uint64_t step, float* g, float* g_m, float* g_v, int32_t* status,
                             cudaStream_t s) {
  const int ngroups = static_cast<int>(K / 16);
  int T = 32;
  while (T < ngroups && T < 256) T <<= 1;
  const int gpt = (ngroups + T - 1) / T;  // 1..8
  const uint32_t sl = static_cast<uint32_t>(seed), sh = static_cast<uint32_t>(seed >> 32);
  const uint32_t tl = static_cast<uint32_t>(step), th = static_cast<uint32_t>(step >> 32);
  const int k = static_cast<int>(K);
  const unsigned grid = static_cast<unsigned>(N);
#define QL_UPD(G, W)                                                                          \
  update_sr_kernel<G, W><<<grid, T, 0, s>>>(wq, sw, grad, k, c, m, v, sl, sh, tl, th, g, g_m, \
                                            g_v, status)
  if (g != nullptr) {  // weight norm: power-of-two thread count for the pinned reduction
    const int64_t row_bytes = K * (c.kind == QL_ADAMW ? 13 : 5);
    // Dynamic budget: the opt-in limit less the kernel's own static arrays.
    static int64_t wn_budget[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && __atomic_load_n(&wn_budget[dev], __ATOMIC_ACQUIRE) == 0) {
      cudaFuncAttributes fa{};
      cudaError_t e = cudaFuncGetAttributes(&fa, update_sr_wn_staged_kernel);
      int64_t b = -1;
      if (e == cudaSuccess) {
        b = device_info().smem_optin - static_cast<int64_t>(fa.sharedSizeBytes);
        e = cudaFuncSetAttribute(update_sr_wn_staged_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(b));
      }
      if (e != cudaSuccess) {
        (void)cudaGetLastError();  // returned here; not left for a later check
        return e;
      }
      __atomic_store_n(&wn_budget[dev], b, __ATOMIC_RELEASE);
    }
    const int64_t budget = dev < 64 ? __atomic_load_n(&wn_budget[dev], __ATOMIC_ACQUIRE) : 0;
    if (row_bytes <= budget) {
      PhiloxKeys keys;
      for (int r = 0; r < 10; ++r) {
        keys.k0[r] = sl + static_cast<uint32_t>(r) * 0x9E3779B9u;
        keys.k1[r] = sh + static_cast<uint32_t>(r) * 0xBB67AE85u;
      }
      const int nch = static_cast<int>(K / 4);
      const int tr = std::max(T, std::min(512, std::max(32, (nch / QL_UPDATE_STAGED_CHUNKS + 31) / 32 * 32)));
      update_sr_wn_staged_kernel<<<grid, tr, static_cast<size_t>(row_bytes), s>>>(
          wq, sw, grad, k, c, m, v, keys, tl, th, g, g_m, g_v, T, status);
      count_launches(1);
      return cudaGetLastError();
    }
    if (gpt <= 1) QL_UPD(1, true);
    else if (gpt <= 2) QL_UPD(2, true);
    else if (gpt <= 4) QL_UPD(4, true);
    else QL_UPD(8, true);
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
      update_sr_staged_kernel<<<grid, tr, static_cast<size_t>(row_bytes), s>>>(
          wq, sw, grad, k, c, m, v, keys, tl, th, status);
      count_launches(1);
      return cudaGetLastError();
    }
    // Longer rows: registers and a parked row of 4 K bytes.
    int tr = (nch + QL_UPDATE_CHUNKS_PER_THREAD - 1) / QL_UPDATE_CHUNKS_PER_THREAD;
    tr = std::min(512, std::max(32, (tr + 31) / 32 * 32));
    static bool smem_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !__atomic_load_n(&smem_set[dev], __ATOMIC_ACQUIRE)) {
      cudaFuncSetAttribute(update_sr_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           4 * 32768);
      __atomic_store_n(&smem_set[dev], true, __ATOMIC_RELEASE);
    }
    update_sr_rows_kernel<<<grid, tr, static_cast<size_t>(4) * K, s>>>(
        wq, sw, grad, k, c, m, v, keys, tl, th, status);
  }
#undef QL_UPD
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ql
