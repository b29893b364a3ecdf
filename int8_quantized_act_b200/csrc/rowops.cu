// rowops.cu - HBM-bound row kernels of the INT8 quantized-training Linear
// layer: per-row symmetric int8 quantization with optional column scaling and
// block-Hadamard rotation (OneTrainer PR #1681 "Int8 conv rot", item 1 and
// summary), the standalone rotation, and the column-wise gradient
// quantization that feeds the weight-gradient GEMM.
//
// Layout: a warp owns 256 consecutive columns of a row ("chunk"), 8 per lane,
// read with 128-bit loads (fp32: two per lane).  A Hadamard block (<= 256)
// never straddles chunks, so the rotation needs only in-lane butterflies and
// warp shuffles.  Rows whose chunks fit in registers are read from HBM once.
#include "launch.h"
#include "rowops.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

template <typename T>
__device__ __forceinline__ const T* row_ptr(const void* base, int64_t r, int64_t ld) {
  return reinterpret_cast<const T*>(base) + r * ld;
}

// ---------------------------------------------------------------------------
// Quantize rows whose chunks fit in registers: WPR warps per row, CPW chunks
// per warp (WPR * CPW * 256 >= cols).  CTA = 8 warps = 8/WPR rows at a time.
template <typename InT, int CPW, int WPR>
__global__ void __launch_bounds__(256) quant_rows_reg_kernel(
    const InT* __restrict__ x, int64_t rows, int cols, int64_t ldx,
    const float* __restrict__ col_scale, int B, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status) {
  constexpr int RPC = 8 / WPR;
  __shared__ float s_max[8];
  __shared__ int s_bad[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp / WPR, wir = warp % WPR;
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * RPC; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.x) * RPC) {
    const int64_t r = r0 + slot;
    const bool rv = r < rows;
    float v[CPW][8];
    float amax = 0.0f;
    int bad = 0;
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int col = (wir + j * WPR) * 256 + lane * 8;
      if (rv && col < cols) {
        load8(x + r * ldx + col, v[j]);
        if (col_scale) {
          float c8[8];
          load8(col_scale + col, c8);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[j][i] = v[j][i] * c8[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
      }
      if (B > 0) fwht_chunk(v[j], B, lane, hc);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        bad |= !finite(v[j][i]);
        amax = fmaxf(amax, fabsf(v[j][i]));
      }
    }
    amax = warp_max(amax);
    bad = warp_or(bad);
    if (WPR > 1) {
      if (lane == 0) {
        s_max[warp] = amax;
        s_bad[warp] = bad;
      }
      __syncthreads();
#pragma unroll
      for (int w = 0; w < WPR; ++w) {
        amax = fmaxf(amax, s_max[slot * WPR + w]);
        bad |= s_bad[slot * WPR + w];
      }
      __syncthreads();
    }
    if (rv) {
      if (amax == 0.0f) {
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const int col = (wir + j * WPR) * 256 + lane * 8;
          if (col < cols) *reinterpret_cast<uint2*>(q + r * ldq + col) = make_uint2(0u, 0u);
        }
        if (wir == 0 && lane == 0) {
          row_scale[r] = 0.0f;
          if (flags & QL_REJECT_ZERO_ROWS) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
        }
      } else {
        const float inv = 127.0f / amax;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const int col = (wir + j * WPR) * 256 + lane * 8;
          if (col < cols) {
            int c[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = code_rne(v[j][i] * inv);
            *reinterpret_cast<uint2*>(q + r * ldq + col) =
                make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
          }
        }
        if (wir == 0 && lane == 0) row_scale[r] = amax / 127.0f;
      }
      if (bad && wir == 0 && lane == 0) atomicOr(status, 1 << QL_ERR_NONFINITE);
    }
  }
}

// ---------------------------------------------------------------------------
// Quantize long rows (more chunks than fit in registers): one CTA per row,
// two passes over the row (the second re-reads it, normally from L2).
template <typename InT>
__global__ void __launch_bounds__(256) quant_rows_stream_kernel(
    const InT* __restrict__ x, int64_t rows, int cols, int64_t ldx,
    const float* __restrict__ col_scale, int B, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status) {
  __shared__ float s_max[8];
  __shared__ int s_bad[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = (cols + 255) / 256;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    float amax = 0.0f;
    int bad = 0;
    for (int ch = warp; ch < nchunks; ch += 8) {
      const int col = ch * 256 + lane * 8;
      float v[8];
      if (col < cols) {
        load8(x + r * ldx + col, v);
        if (col_scale) {
          float c8[8];
          load8(col_scale + col, c8);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = v[i] * c8[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      }
      if (B > 0) fwht_chunk(v, B, lane, hc);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        bad |= !finite(v[i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
    }
    amax = warp_max(amax);
    bad = warp_or(bad);
    if (lane == 0) {
      s_max[warp] = amax;
      s_bad[warp] = bad;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      amax = fmaxf(amax, s_max[w]);
      bad |= s_bad[w];
    }
    __syncthreads();
    const float inv = amax == 0.0f ? 0.0f : 127.0f / amax;
    for (int ch = warp; ch < nchunks; ch += 8) {
      const int col = ch * 256 + lane * 8;
      float v[8];
      if (col < cols) {
        load8(x + r * ldx + col, v);
        if (col_scale) {
          float c8[8];
          load8(col_scale + col, c8);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = v[i] * c8[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      }
      if (B > 0) fwht_chunk(v, B, lane, hc);
      if (col < cols) {
        int c[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = amax == 0.0f ? 0 : code_rne(v[i] * inv);
        *reinterpret_cast<uint2*>(q + r * ldq + col) =
            make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
      }
    }
    if (threadIdx.x == 0) {
      row_scale[r] = amax == 0.0f ? 0.0f : amax / 127.0f;
      if (amax == 0.0f && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
      if (bad) atomicOr(status, 1 << QL_ERR_NONFINITE);
    }
  }
}

// ---------------------------------------------------------------------------
// y = x R: each warp rotates one 256-column chunk at a time.
template <typename InT, typename OutT>
__global__ void __launch_bounds__(256) hadamard_kernel(const InT* x, int64_t ldx, OutT* y,
                                                       int64_t ldy, int64_t rows, int cols,
                                                       int B, float hc) {
  const int lane = threadIdx.x & 31;
  const int64_t nchunks = (cols + 255) / 256;
  const int64_t total = rows * nchunks;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); t < total;
       t += wstride) {
    const int64_t r = t / nchunks;
    const int col = static_cast<int>(t % nchunks) * 256 + lane * 8;
    float v[8];
    if (col < cols) {
      // x may alias y: plain (not read-only cached) loads.
      const InT* p = x + r * ldx + col;
      if constexpr (sizeof(InT) == 4) {
        const float4 a = reinterpret_cast<const float4*>(p)[0];
        const float4 b = reinterpret_cast<const float4*>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = __uint_as_float(w[i] << 16);
          v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    fwht_chunk(v, B, lane, hc);
    if (col < cols) store8(y + r * ldy + col, v);
  }
}

// ---------------------------------------------------------------------------
// Column statistics for the weight-gradient quantization.  Block = 8 warps
// over one 256-column chunk and a slab of rows; lane owns 8 columns.
constexpr int kColSlab = 128;

template <typename InT>
__global__ void __launch_bounds__(256) colstats_kernel(const InT* __restrict__ dy, int64_t M,
                                                       int N, const float* __restrict__ sx,
                                                       uint32_t* __restrict__ colmax,
                                                       double* __restrict__ colsum,
                                                       int32_t* __restrict__ status) {
  __shared__ float s_max[8][256];
  __shared__ double s_sum[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * 256 + lane * 8;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kColSlab;
  const int64_t m1 = m0 + kColSlab < M ? m0 + kColSlab : M;
  float mx[8];
  double sm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mx[i] = 0.0f;
    sm[i] = 0.0;
  }
  int bad = 0;
  if (col < N) {
    for (int64_t m = m0 + warp; m < m1; m += 8) {
      float d[8];
      load8(dy + m * N + col, d);
      const float s = __ldg(sx + m);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = d[i] * s;
        bad |= !finite(t);
        mx[i] = fmaxf(mx[i], fabsf(t));
        sm[i] += static_cast<double>(d[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_max[warp][lane * 8 + i] = mx[i];
    s_sum[warp][lane * 8 + i] = sm[i];
  }
  bad = warp_or(bad);
  if (bad && lane == 0) atomicOr(status, 1 << QL_ERR_NONFINITE);
  __syncthreads();
  const int c = threadIdx.x;  // one column per thread
  if (blockIdx.x * 256 + c < N) {
    float a = 0.0f;
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      a = fmaxf(a, s_max[w][c]);
      t += s_sum[w][c];
    }
    // max of non-negative floats = max of their bit patterns
    atomicMax(colmax + blockIdx.x * 256 + c, __float_as_uint(a));
    atomicAdd(colsum + blockIdx.x * 256 + c, t);
  }
}

__global__ void colfinalize_kernel(const uint32_t* __restrict__ colmax,
                                   const double* __restrict__ colsum, int N, float* s2,
                                   float* inv2, float* db) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const float amax = __uint_as_float(colmax[n]);
  s2[n] = amax == 0.0f ? 0.0f : amax / 127.0f;
  inv2[n] = amax == 0.0f ? 0.0f : 127.0f / amax;
  if (db) db[n] = static_cast<float>(colsum[n]);
}

// One thread per 16 consecutive columns of one row.
template <typename InT>
__global__ void __launch_bounds__(256) colquant_kernel(const InT* __restrict__ dy, int64_t M,
                                                       int N, const float* __restrict__ sx,
                                                       const float* __restrict__ inv2,
                                                       int8_t* __restrict__ q) {
  const int per_row = N / 16;
  const int64_t total = M * per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = t / per_row;
    const int col = static_cast<int>(t % per_row) * 16;
    float d0[8], d1[8], i0[8], i1[8];
    load8(dy + m * N + col, d0);
    load8(dy + m * N + col + 8, d1);
    load8(inv2 + col, i0);
    load8(inv2 + col + 8, i1);
    const float s = __ldg(sx + m);
    int c[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = code_rne((d0[i] * s) * i0[i]);
      c[8 + i] = code_rne((d1[i] * s) * i1[i]);
    }
    *reinterpret_cast<uint4*>(q + m * N + col) =
        make_uint4(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]),
                   pack4(c[8], c[9], c[10], c[11]), pack4(c[12], c[13], c[14], c[15]));
  }
}

template <typename OutT>
__global__ void fill_rows_kernel(OutT* out, int64_t rows, int cols, const float* bias) {
  const int64_t total = rows * cols;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float b = bias ? bias[t % cols] : 0.0f;
    if constexpr (sizeof(OutT) == 4) {
      out[t] = b;
    } else {
      out[t] = __float2bfloat16_rn(b);
    }
  }
}

int grid_cap(int64_t want, int per_sm) {
  const int64_t cap = static_cast<int64_t>(device_info().sms) * per_sm;
  if (want < 1) want = 1;
  return static_cast<int>(want < cap ? want : cap);
}

template <typename InT>
cudaError_t quant_rows_t(const void* xv, int64_t rows, int64_t cols, int64_t ldx,
                         const float* cs, int B, float hc, unsigned flags, int8_t* q, int64_t ldq,
                         float* rs, int32_t* st, cudaStream_t s) {
  const InT* x = reinterpret_cast<const InT*>(xv);
  const int nch = static_cast<int>((cols + 255) / 256);
  const int c = static_cast<int>(cols);
  if (nch <= 64) {
    const int wpr = nch <= 1 ? 1 : nch <= 2 ? 2 : nch <= 4 ? 4 : 8;
    const int cpw = (nch + wpr - 1) / wpr;  // 1..8
    const int rpc = 8 / wpr;
    const int grid = grid_cap((rows + rpc - 1) / rpc, 8);
#define QL_QR(CPW, WPR)                                                                       \
  quant_rows_reg_kernel<InT, CPW, WPR><<<grid, 256, 0, s>>>(x, rows, c, ldx, cs, B, hc, flags, \
                                                             q, ldq, rs, st)
    if (wpr == 1) QL_QR(1, 1);
    else if (wpr == 2) QL_QR(1, 2);
    else if (wpr == 4) QL_QR(1, 4);
    else if (cpw <= 1) QL_QR(1, 8);
    else if (cpw <= 2) QL_QR(2, 8);
    else if (cpw <= 4) QL_QR(4, 8);
    else QL_QR(8, 8);
#undef QL_QR
  } else {
    const int grid = grid_cap(rows, 8);
    quant_rows_stream_kernel<InT><<<grid, 256, 0, s>>>(x, rows, c, ldx, cs, B, hc, flags, q, ldq,
                                                       rs, st);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_rows(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                              const float* col_scale, int B, float hc, unsigned flags,
                              int8_t* q, int64_t ldq, float* row_scale, int32_t* status,
                              cudaStream_t s) {
  if (xt == QL_BF16)
    return quant_rows_t<__nv_bfloat16>(x, rows, cols, ldx, col_scale, B, hc, flags, q, ldq,
                                       row_scale, status, s);
  return quant_rows_t<float>(x, rows, cols, ldx, col_scale, B, hc, flags, q, ldq, row_scale,
                             status, s);
}

cudaError_t launch_hadamard(const void* x, int xt, int64_t ldx, void* y, int yt, int64_t ldy,
                            int64_t rows, int64_t cols, int B, float hc, cudaStream_t s) {
  const int64_t tasks = rows * ((cols + 255) / 256);
  const int grid = grid_cap((tasks + 7) / 8, 8);
  const int c = static_cast<int>(cols);
#define QL_HD(IT, OT)                                                                        \
  hadamard_kernel<IT, OT><<<grid, 256, 0, s>>>(reinterpret_cast<const IT*>(x), ldx,          \
                                               reinterpret_cast<OT*>(y), ldy, rows, c, B, hc)
  if (xt == QL_F32 && yt == QL_F32) QL_HD(float, float);
  else if (xt == QL_F32) QL_HD(float, __nv_bfloat16);
  else if (yt == QL_F32) QL_HD(__nv_bfloat16, float);
  else QL_HD(__nv_bfloat16, __nv_bfloat16);
#undef QL_HD
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_colstats(const void* dy, int dyt, int64_t M, int64_t N, const float* sx,
                            uint32_t* colmax, double* colsum, int32_t* status, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((N + 255) / 256),
                  static_cast<unsigned>((M + kColSlab - 1) / kColSlab));
  if (dyt == QL_BF16)
    colstats_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(dy), M, static_cast<int>(N), sx, colmax, colsum,
        status);
  else
    colstats_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(dy), M,
                                                static_cast<int>(N), sx, colmax, colsum, status);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_colfinalize(const uint32_t* colmax, const double* colsum, int64_t N,
                               float* s2, float* inv2, float* db, cudaStream_t s) {
  colfinalize_kernel<<<static_cast<unsigned>((N + 255) / 256), 256, 0, s>>>(
      colmax, colsum, static_cast<int>(N), s2, inv2, db);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_colquant(const void* dy, int dyt, int64_t M, int64_t N, const float* sx,
                            const float* inv2, int8_t* q, cudaStream_t s) {
  const int64_t items = M * (N / 16);
  const int grid = grid_cap((items + 255) / 256, 8);
  if (dyt == QL_BF16)
    colquant_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(dy), M, static_cast<int>(N), sx, inv2, q);
  else
    colquant_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(dy), M,
                                                static_cast<int>(N), sx, inv2, q);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fill_rows(void* out, int ot, int64_t rows, int64_t cols, const float* bias,
                             cudaStream_t s) {
  const int grid = grid_cap((rows * cols + 255) / 256, 8);
  if (ot == QL_BF16)
    fill_rows_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        reinterpret_cast<__nv_bfloat16*>(out), rows, static_cast<int>(cols), bias);
  else
    fill_rows_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<float*>(out), rows,
                                                 static_cast<int>(cols), bias);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ql
