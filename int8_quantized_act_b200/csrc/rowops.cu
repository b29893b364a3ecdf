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
#include <algorithm>

#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
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
// The row max is carried as |x| bit patterns (abs_bits), which also flags
// inf/NaN; codes are rounded through the float adder (rne_bits).
template <typename InT, int CPW, int WPR>
__global__ void __launch_bounds__(256) quant_rows_reg_kernel(
    const InT* __restrict__ x, int64_t rows, int cols, int64_t ldx,
    const float* __restrict__ col_scale, int B, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status) {
  constexpr int RPC = 8 / WPR;
  __shared__ uint32_t s_max[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp / WPR, wir = warp % WPR;
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * RPC; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.x) * RPC) {
    const int64_t r = r0 + slot;
    const bool rv = r < rows;
    float v[CPW][8];
    uint32_t mbits = 0;
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int chunk0 = (wir + j * WPR) * 256;  // same for the whole warp
      const int col = chunk0 + lane * 8;
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
      if (B > 0 && rv && chunk0 < cols) fwht_chunk(v[j], B, lane, hc);
#pragma unroll
      for (int i = 0; i < 8; ++i) mbits = max(mbits, abs_bits(v[j][i]));
    }
    mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
    if (WPR > 1) {
      if (lane == 0) s_max[warp] = mbits;
      __syncthreads();
#pragma unroll
      for (int w = 0; w < WPR; ++w) mbits = max(mbits, s_max[slot * WPR + w]);
      __syncthreads();
    }
    if (rv) {
      const float amax = __uint_as_float(mbits);
      const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int col = (wir + j * WPR) * 256 + lane * 8;
        if (col < cols) {
          uint32_t b[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) b[i] = rne_bits_prod(v[j][i], inv);
          *reinterpret_cast<uint2*>(q + r * ldq + col) =
              make_uint2(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]));
        }
      }
      if (wir == 0 && lane == 0) {
        row_scale[r] = mbits == 0 ? 0.0f : amax / 127.0f;
        if (mbits == 0 && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
        if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Quantize rows staged in shared memory by the bulk-copy engine: a persistent
// CTA (8 warps) walks rows r = blockIdx.x + i * gridDim.x through a ring of
// `stages` row buffers, so several rows per CTA are in flight without holding
// registers; each warp then takes chunks wir, wir + 8, ... (CPW of them) of the
// staged row, exactly as the register kernel does.  Waits are bounded: on a
// time-out the CTA reports QL_ERR_TIMEOUT, lets its copies land and returns.
// BT: 0 = no rotation, > 0 = block size fixed at compile time, < 0 = block
// size B given at run time.
template <typename InT, int CPW, int BT>
__global__ void __launch_bounds__(256) quant_rows_tma_kernel(
    const InT* __restrict__ x, int64_t rows, int cols, int64_t ldx,
    const float* __restrict__ col_scale, int B, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status, int stages, int stage_bytes) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t s_max[8];
  __shared__ __align__(8) uint64_t s_full[8];
  __shared__ volatile int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t row_bytes = static_cast<uint32_t>(cols) * sizeof(InT);
  const int64_t mine = rows > blockIdx.x ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) mbar_init(smem_u32(&s_full[st]), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages && st < mine; ++st) {
      const int64_t r = blockIdx.x + static_cast<int64_t>(st) * gridDim.x;
      mbar_arrive_expect_tx(smem_u32(&s_full[st]), row_bytes);
      bulk_load(smem_u32(smem + st * stage_bytes), x + r * ldx, row_bytes, smem_u32(&s_full[st]));
    }
  }
  // A lane owns the same columns in every row: keep their scales in registers.
  float cs[CPW][8];
#pragma unroll
  for (int j = 0; j < CPW; ++j) {
    const int col = (warp + 8 * j) * 256 + lane * 8;
    if (col_scale && col < cols) {
      load8(col_scale + col, cs[j]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[j][e] = 1.0f;
    }
  }
  int64_t done = 0;
  for (int64_t i = 0; i < mine; ++i) {
    const int st = static_cast<int>(i % stages);
    const uint32_t parity = static_cast<uint32_t>((i / stages) & 1);
    const int64_t r = blockIdx.x + i * gridDim.x;
    // A thread that gives up (mbar_wait raises s_abort) still takes part in
    // both barriers below; the CTA leaves the loop together after the second.
    const bool ok = mbar_wait(smem_u32(&s_full[st]), parity, &s_abort);
    const InT* xs = reinterpret_cast<const InT*>(smem + st * stage_bytes);
    float v[CPW][8];
    uint32_t mbits = 0;
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int chunk0 = (warp + 8 * j) * 256;
      const int col = chunk0 + lane * 8;
      if (ok && col < cols) {
        if constexpr (sizeof(InT) == 4) {
          const float4 a = reinterpret_cast<const float4*>(xs + col)[0];
          const float4 b = reinterpret_cast<const float4*>(xs + col)[1];
          v[j][0] = a.x; v[j][1] = a.y; v[j][2] = a.z; v[j][3] = a.w;
          v[j][4] = b.x; v[j][5] = b.y; v[j][6] = b.z; v[j][7] = b.w;
        } else {
          const uint4 u = *reinterpret_cast<const uint4*>(xs + col);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[j][2 * e] = __uint_as_float(w4[e] << 16);
            v[j][2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
          }
        }
        if (col_scale) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[j][e] = v[j][e] * cs[j][e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[j][e] = 0.0f;
      }
      if constexpr (BT > 0) {
        if (chunk0 < cols) fwht_chunk_ct<BT>(v[j], lane, hc);
      } else if constexpr (BT < 0) {
        if (chunk0 < cols) fwht_chunk(v[j], B, lane, hc);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) mbits = max(mbits, abs_bits(v[j][e]));
    }
    mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
    if (lane == 0) s_max[warp] = mbits;
    __syncthreads();  // every thread is done reading stage st
    if (threadIdx.x == 0 && i + stages < mine && !s_abort) {
      fence_proxy_async_smem();
      const int64_t rn = blockIdx.x + (i + stages) * gridDim.x;
      mbar_arrive_expect_tx(smem_u32(&s_full[st]), row_bytes);
      bulk_load(smem_u32(smem + st * stage_bytes), x + rn * ldx, row_bytes, smem_u32(&s_full[st]));
    }
#pragma unroll
    for (int w = 0; w < 8; ++w) mbits = max(mbits, s_max[w]);
    __syncthreads();  // s_max may be rewritten by the next row
    if (s_abort) break;
    const float amax = __uint_as_float(mbits);
    const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int col = (warp + 8 * j) * 256 + lane * 8;
      if (col < cols) *reinterpret_cast<uint2*>(q + r * ldq + col) = codes8(v[j], inv);
    }
    if (threadIdx.x == 0) {
      row_scale[r] = mbits == 0 ? 0.0f : amax / 127.0f;
      if (mbits == 0 && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
      if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
    }
    done = i + 1;
  }
  if (threadIdx.x == 0 && s_abort) {
    // Timed out: let every copy already issued (rows done .. done+stages-1)
    // land before the CTA exits.
    atomicOr(status, 1 << QL_ERR_TIMEOUT);
    for (int64_t i = done; i < mine && i < done + stages; ++i)
      mbar_wait_drain(smem_u32(&s_full[i % stages]), static_cast<uint32_t>((i / stages) & 1));
  }
}

// ---------------------------------------------------------------------------
constexpr int kWideStagesMax = 4;

// The block-128 rotation + quantization of bf16 rows (the forward's input).
// A row's cols/128 blocks are spread over 4 lanes each, 32 columns per lane,
// so five of the seven butterfly stages stay inside a lane and two use
// shuffles (the 256-column layout above needs four).  The two rows of a pair
// are laid end to end over the CTA's lanes (a warp may hold the end of one
// row and the start of the next; a 4-lane block never straddles a warp), so
// few lanes idle.  Pairs of rows arrive by one TMA load per stage from a
// [rows][cols/64][64] view with the 128-byte swizzle, which puts each lane's
// four 16-byte pieces in distinct banks.
__global__ void __launch_bounds__(512, 2) quant_b128_wide_kernel(
    const __grid_constant__ CUtensorMap tm, int64_t rows, int cols, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status, int stages, int stage_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint32_t s_max[2][16][2];  // [pair parity][warp][row of the pair]
  __shared__ __align__(8) uint64_t s_full[kWideStagesMax];
  __shared__ volatile int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int lines = cols >> 6;      // 128-byte lines per row
  const int row_lanes = cols >> 5;  // 4 lanes per 128-column block
  const int sub = static_cast<int>(threadIdx.x) / row_lanes;  // row of the pair; 2: idle lane
  const int j = static_cast<int>(threadIdx.x) - sub * row_lanes;
  const int col0 = (j >> 2) * 128 + (j & 3) * 32;
  const bool active = sub < 2;
  const int64_t pairs = (rows + 1) >> 1;
  const int64_t mine = pairs > blockIdx.x ? (pairs - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) mbar_init(smem_u32(&s_full[st]), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm);
    for (int st = 0; st < stages && st < mine; ++st) {
      const int64_t p = blockIdx.x + static_cast<int64_t>(st) * gridDim.x;
      mbar_arrive_expect_tx(smem_u32(&s_full[st]), static_cast<uint32_t>(2 * lines * 128));
      tma_load_3d(smem_u32(smem + st * stage_bytes), &tm, smem_u32(&s_full[st]), 0, 0,
                  static_cast<int>(2 * p));
    }
  }
  int64_t done = 0;
  for (int64_t i = 0; i < mine; ++i) {
    const int st = static_cast<int>(i % stages);
    const uint32_t parity = static_cast<uint32_t>((i / stages) & 1);
    const int64_t r = 2 * (blockIdx.x + i * gridDim.x) + sub;
    // A thread that gives up (mbar_wait raises s_abort) still takes part in
    // the barrier below; the CTA leaves the loop together after it.
    const bool ok = mbar_wait(smem_u32(&s_full[st]), parity, &s_abort);
    float v[32];
    if (ok && active) {
      // Lane's 64 bytes are half of line gl = sub*lines + col0/64; piece p
      // (16 bytes) sits at 16-byte slot (4*half + p) ^ (gl & 7) of the line.
      const int gl = sub * lines + (col0 >> 6);
      const int half = (col0 >> 5) & 1;
      const uint8_t* line = smem + st * stage_bytes + gl * 128;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        const uint4 u = *reinterpret_cast<const uint4*>(line + (((half << 2) + pc) ^ (gl & 7)) * 16);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * pc + 2 * e] = __uint_as_float(w4[e] << 16);
          v[8 * pc + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0.0f;
    }
    fwht128_wide(v, lane, hc);
    uint32_t mbits = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) mbits = max(mbits, abs_bits(v[e]));
    const uint32_t m0 = __reduce_max_sync(0xFFFFFFFFu, sub == 0 ? mbits : 0u);
    const uint32_t m1 = __reduce_max_sync(0xFFFFFFFFu, sub == 1 ? mbits : 0u);
    uint32_t(*smax)[2] = s_max[i & 1];
    if (lane == 0) {
      smax[warp][0] = m0;
      smax[warp][1] = m1;
    }
    // Every thread is done reading stage st (and, one pair back, the other
    // half of s_max, which the next pair rewrites).
    __syncthreads();
    if (threadIdx.x == 0 && i + stages < mine && !s_abort) {
      fence_proxy_async_smem();
      const int64_t pn = blockIdx.x + (i + stages) * gridDim.x;
      mbar_arrive_expect_tx(smem_u32(&s_full[st]), static_cast<uint32_t>(2 * lines * 128));
      tma_load_3d(smem_u32(smem + st * stage_bytes), &tm, smem_u32(&s_full[st]), 0, 0,
                  static_cast<int>(2 * pn));
    }
    if (s_abort) break;
    if (active && r < rows) {
      mbits = 0;
      for (int w = 0; w < nwarps; ++w) mbits = max(mbits, smax[w][sub]);
      const float amax = __uint_as_float(mbits);
      const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
      uint32_t b[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) b[e] = rne_bits_prod(v[e], inv);
      uint4* dst = reinterpret_cast<uint4*>(q + r * ldq + col0);
      dst[0] = make_uint4(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]),
                          pack_codes(b[8], b[9], b[10], b[11]), pack_codes(b[12], b[13], b[14], b[15]));
      dst[1] = make_uint4(pack_codes(b[16], b[17], b[18], b[19]), pack_codes(b[20], b[21], b[22], b[23]),
                          pack_codes(b[24], b[25], b[26], b[27]), pack_codes(b[28], b[29], b[30], b[31]));
      if (j == 0) {
        row_scale[r] = mbits == 0 ? 0.0f : amax / 127.0f;
        if (mbits == 0 && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
        if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
      }
    }
    done = i + 1;
  }
  if (threadIdx.x == 0 && s_abort) {
    atomicOr(status, 1 << QL_ERR_TIMEOUT);
    for (int64_t i = done; i < mine && i < done + stages; ++i)
      mbar_wait_drain(smem_u32(&s_full[i % stages]), static_cast<uint32_t>((i / stages) & 1));
  }
}

// ---------------------------------------------------------------------------
// Quantize long rows (more chunks than fit in registers): one CTA per row,
// two passes over the row (the second re-reads it, normally from L2).
template <typename InT>
__device__ __forceinline__ void load_chunk(const InT* xr, const float* cs, int col, int cols,
                                           float (&v)[8]) {
  if (col < cols) {
    load8(xr + col, v);
    if (cs) {
      float c8[8];
      load8(cs + col, c8);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = v[i] * c8[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
}

template <typename InT>
__global__ void __launch_bounds__(256) quant_rows_stream_kernel(
    const InT* __restrict__ x, int64_t rows, int cols, int64_t ldx,
    const float* __restrict__ col_scale, int B, float hc, unsigned flags,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ row_scale,
    int32_t* __restrict__ status) {
  __shared__ uint32_t s_max[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = (cols + 255) / 256;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    uint32_t mbits = 0;
    for (int ch = warp; ch < nchunks; ch += 8) {
      float v[8];
      load_chunk(x + r * ldx, col_scale, ch * 256 + lane * 8, cols, v);
      if (B > 0) fwht_chunk(v, B, lane, hc);
#pragma unroll
      for (int i = 0; i < 8; ++i) mbits = max(mbits, abs_bits(v[i]));
    }
    mbits = __reduce_max_sync(0xFFFFFFFFu, mbits);
    if (lane == 0) s_max[warp] = mbits;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 8; ++w) mbits = max(mbits, s_max[w]);
    __syncthreads();
    const float amax = __uint_as_float(mbits);
    const float inv = mbits == 0 ? 0.0f : 127.0f / amax;
    for (int ch = warp; ch < nchunks; ch += 8) {
      const int col = ch * 256 + lane * 8;
      float v[8];
      load_chunk(x + r * ldx, col_scale, col, cols, v);
      if (B > 0) fwht_chunk(v, B, lane, hc);
      if (col < cols) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = rne_bits_prod(v[i], inv);
        *reinterpret_cast<uint2*>(q + r * ldq + col) =
            make_uint2(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]));
      }
    }
    if (threadIdx.x == 0) {
      row_scale[r] = mbits == 0 ? 0.0f : amax / 127.0f;
      if (mbits == 0 && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
      if (mbits >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
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

// w[r, :] = s[r] * q[r, :] (one float32 multiply), then for B > 0 the
// block-Hadamard of fwht_chunk (R is its own inverse: back to the original
// basis).  A warp converts one 256-column chunk, 8 codes per lane.
template <typename OutT>
__global__ void __launch_bounds__(256) dequant_rows_kernel(const int8_t* __restrict__ q,
                                                           int64_t ldq, const float* __restrict__ s,
                                                           OutT* __restrict__ w, int64_t ldw,
                                                           int64_t rows, int cols, int B, float hc) {
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
      const float sr = s ? __ldg(s + r) : 1.0f;
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(q + r * ldq + col));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t word = i < 4 ? u.x : u.y;
        const int code = static_cast<int8_t>((word >> (8 * (i & 3))) & 0xFFu);
        v[i] = static_cast<float>(code) * sr;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    if (B > 0) fwht_chunk(v, B, lane, hc);
    if (col < cols) store8(w + r * ldw + col, v);
  }
}


// Zero the column maxima and sums and (if given) the row maxima before the
// column statistics pass accumulates into them: one launch for all three.
__global__ void zero_stats_kernel(uint32_t* __restrict__ colmax, double* __restrict__ colsum,
                                  int64_t N, uint32_t* __restrict__ rowmax, int64_t M) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N + M; i += stride) {
    if (i < N) {
      colmax[i] = 0u;
      colsum[i] = 0.0;
    } else if (rowmax) {
      rowmax[i - N] = 0u;
    }
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
  const int64_t row_bytes = cols * static_cast<int64_t>(sizeof(InT));
  if (sizeof(InT) == 2 && quant_blk_eligible(rows, cols, ldx, B, cs != nullptr))
    return launch_quant_blk(x, rows, cols, ldx, B, hc, flags, q, ldq, rs, st, s);
  if (sizeof(InT) == 2 && B == 128 && !cs && cols % 128 == 0 && cols >= 1024 && cols <= 8192 &&
      (ldx * 2) % 16 == 0 && rows >= 4 * device_info().sms) {
    CUtensorMap tm;
    if (!encode_rows_128b(&tm, 2, x, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                          static_cast<uint64_t>(ldx) * 2, 2))
      return cudaErrorInvalidValue;
    // Two rows' blocks (4 lanes each) over whole warps; CTAs per SM from the
    // kernel's actual occupancy, three stages each.
    const int threads = static_cast<int>((2 * (cols / 128) * 4 + 31) / 32 * 32);
    const int stage_bytes = static_cast<int>((2 * row_bytes + 1023) / 1024 * 1024);
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && __atomic_load_n(&occ[dev], __ATOMIC_ACQUIRE) == 0) {
      cudaFuncSetAttribute(quant_b128_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 110000);
      __atomic_store_n(&occ[dev], -1, __ATOMIC_RELEASE);
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_b128_wide_kernel, threads,
                                                      3 * stage_bytes + 1024) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    per_sm = std::min(per_sm, 3);
    int stages = (220000 / per_sm - 2048) / stage_bytes;
    stages = stages < 2 ? 2 : stages > kWideStagesMax ? kWideStagesMax : stages;
    const int smem = stages * stage_bytes + 1024;
    const int64_t pairs = (rows + 1) / 2;
    const int grid = static_cast<int>(std::min<int64_t>(pairs, static_cast<int64_t>(device_info().sms) * per_sm));
    quant_b128_wide_kernel<<<grid, threads, smem, s>>>(tm, rows, c, hc, flags, q, ldq, rs, st,
                                                        stages, stage_bytes);
    count_launches(1);
    return cudaGetLastError();
  }
  if (nch >= 9 && nch <= 32 && rows >= 2 * device_info().sms) {
    // Rows of 2304..8192 columns, enough of them to fill the GPU: bulk-copy
    // staged kernel, 2-4 rows per CTA in flight within ~96 KB.
    const int stage_bytes = static_cast<int>((row_bytes + 127) / 128 * 128);
    int stages = 98304 / stage_bytes;
    stages = stages < 2 ? 2 : stages > 4 ? 4 : stages;
    const int smem = stages * stage_bytes;
    const int per_sm = 200000 / (smem + 2048) > 4 ? 4 : 200000 / (smem + 2048);
    const int grid = grid_cap(rows, per_sm < 1 ? 1 : per_sm);
    const int cpw = (nch + 7) / 8;
#define QL_QT(CPW, BT)                                                                         \
  do {                                                                                         \
    static bool attr_set[64] = {false};                                                        \
    int dev = 0;                                                                               \
    cudaGetDevice(&dev);                                                                       \
    if (dev < 64 && !__atomic_load_n(&attr_set[dev], __ATOMIC_ACQUIRE)) {                      \
      cudaFuncSetAttribute(quant_rows_tma_kernel<InT, CPW, BT>,                                \
                           cudaFuncAttributeMaxDynamicSharedMemorySize, 100000);               \
      __atomic_store_n(&attr_set[dev], true, __ATOMIC_RELEASE);                                \
    }                                                                                          \
    quant_rows_tma_kernel<InT, CPW, BT><<<grid, 256, smem, s>>>(                               \
        x, rows, c, ldx, cs, B, hc, flags, q, ldq, rs, st, stages, stage_bytes);               \
  } while (0)
#define QL_QT_B(CPW)                  \
  do {                                \
    if (B == 0) QL_QT(CPW, 0);        \
    else if (B == 128) QL_QT(CPW, 128); \
    else QL_QT(CPW, -1);              \
  } while (0)
    if (cpw <= 2) QL_QT_B(2);
    else if (cpw <= 3) QL_QT_B(3);
    else QL_QT_B(4);
#undef QL_QT_B
#undef QL_QT
  } else if (nch <= 64) {
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
    else if (cpw <= 3) QL_QR(3, 8);
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

cudaError_t launch_dequant_rows(const int8_t* q, int64_t ldq, const float* s, void* w, int wt,
                                int64_t ldw, int64_t rows, int64_t cols, int B, float hc,
                                cudaStream_t st) {
  const int64_t tasks = rows * ((cols + 255) / 256);
  const int grid = grid_cap((tasks + 7) / 8, 8);
  const int c = static_cast<int>(cols);
  if (wt == QL_BF16)
    dequant_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        q, ldq, s, reinterpret_cast<__nv_bfloat16*>(w), ldw, rows, c, B, hc);
  else
    dequant_rows_kernel<float><<<grid, 256, 0, st>>>(q, ldq, s, reinterpret_cast<float*>(w), ldw,
                                                      rows, c, B, hc);
  count_launches(1);
  return cudaGetLastError();
}


cudaError_t launch_zero_stats(uint32_t* colmax, double* colsum, int64_t N, uint32_t* rowmax,
                              int64_t M, cudaStream_t s) {
  const int64_t n = N + (rowmax ? M : 0);
  const cudaError_t e = launch_pdl(zero_stats_kernel, dim3(grid_cap((n + 255) / 256, 4)), dim3(256),
                                   0, s, colmax, colsum, N, rowmax, rowmax ? M : 0);
  count_launches(1);
  return e == cudaSuccess ? cudaGetLastError() : e;
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
