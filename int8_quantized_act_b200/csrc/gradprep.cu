// gradprep.cu - the gradient quantizations of the backward pass, streamed
// through shared memory by the tensor-memory-access (TMA) engine.
//
// The backward formulas (dX = s'[m] * quant_row(dY * s_w[n]) W_q and
// dW = s''[n] * quant_col(dY * s_x[m])^T X_q) need, per column n, the max over
// m of |dY * s_x| and, per row m, the max over n of |dY * s_w|, before any code
// can be written.  Pass 1 (colstats) gathers the column maxima, the column
// sums (the bias gradient) and, optionally, the row maxima; pass 2
// (dualquant) writes one or both int8 code sets elementwise.
//
// Both passes stream dY in tiles of 1024 columns x 16 rows (bf16) or 8 rows
// (float32), 32 KB each, through a 3-stage ring: a producer warp issues one
// TMA load per 256-column quarter of a tile (rows / columns past the matrix
// read as zero; quarters wholly past the last column are not loaded), so
// each row of a tile is read as 2 KB in a row, while 8 consumer warps work on
// earlier tiles: warp w takes quarter w % 4 and half w / 4 of the rows, 8 (4)
// rows.  Up to 96 KB per CTA and two CTAs per SM are in flight without tying
// up registers.  Block (x, y) owns column block x and a contiguous run of row
// tiles, so per-column state stays in registers.  The per-row factors of a
// warp's rows are loaded one row per lane and broadcast by shuffles.
#include <cuda.h>
#include <cuda_bf16.h>

#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

constexpr int kCols = 256;        // columns of a quarter (8 per lane)
constexpr int kSub = 4;           // quarters per tile
constexpr int kBlockCols = kSub * kCols;
constexpr int kStages = 3;
constexpr int kTileBytes = 32768;
constexpr int kThreads = 288;     // 8 consumer warps + 1 producer warp

template <typename InT>
struct Tile {
  static constexpr int kRows = kTileBytes / (kBlockCols * static_cast<int>(sizeof(InT)));  // 16 / 8
  static constexpr int kRowsPerWarp = kRows / (8 / kSub);                                    // 8 / 4
  static_assert(kRowsPerWarp % 2 == 0 && kRowsPerWarp <= 32, "rows of a warp: pairs, one per lane");
};

// 8 consecutive elements of a staged row as float32, read with 16-byte
// shared-memory loads from a shared-space address.
template <typename InT>
__device__ __forceinline__ void smem_load8(uint32_t addr, float (&v)[8]) {
  if constexpr (sizeof(InT) == 4) {
    const uint4 a = lds128(addr), b = lds128(addr + 16);
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
    v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
  } else {
    const uint4 u = lds128(addr);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(w[e] << 16);
      v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
}

// The ring shared by both passes: tiles t0 .. t1-1 (row tiles) of column
// block cb.  run() calls body(tile, stage_ptr) on the consumer warps for every
// tile in order; the producer warp keeps up to kStages tiles in flight.
struct Ring {
  uint8_t* buf;
  uint64_t* full;
  uint64_t* empty;
  volatile int* abort_flag;

  __device__ void init(int tid) {
    if (tid == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(smem_u32(&full[s]), 1);
        mbar_init(smem_u32(&empty[s]), 8);
      }
      *abort_flag = 0;
      fence_mbar_init();
    }
  }

  // Producer (one thread): load tile t of column block cb into each free
  // stage, the first nsub quarters (those that start before the last column);
  // tiles t0 .. t1-1 in increasing order, or decreasing with rev.
  __device__ void produce(const CUtensorMap* tm, int cb, int nsub, int t0, int t1,
                          int rows_per_tile, bool rev = false) {
    uint32_t issued = 0, issued_phase = 0;
    for (int k = 0; k < t1 - t0; ++k) {
      const int t = rev ? t1 - 1 - k : t0 + k;
      const int s = k % kStages;
      const uint32_t ph = static_cast<uint32_t>(k / kStages) & 1u;
      if (k >= kStages && !mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag)) break;
      mbar_arrive_expect_tx(smem_u32(&full[s]), static_cast<uint32_t>(nsub * (kTileBytes / kSub)));
      for (int q = 0; q < nsub; ++q)
        tma_load_2d(smem_u32(buf + s * kTileBytes + q * (kTileBytes / kSub)), tm,
                    smem_u32(&full[s]), cb * kBlockCols + q * kCols, t * rows_per_tile);
      issued |= 1u << s;
      issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
    }
    // Every copy issued must land before the CTA may exit.
    for (int s = 0; s < kStages; ++s)
      if (issued & (1u << s)) mbar_wait_drain(smem_u32(&full[s]), (issued_phase >> s) & 1u);
  }

  // Consumer warp: wait for tile k, run body, release the stage (the
  // producer's tile order).
  template <typename F>
  __device__ void consume(int t0, int t1, int lane, F&& body, bool rev = false) {
    const uint32_t base = smem_u32(buf);
    for (int k = 0; k < t1 - t0; ++k) {
      const int t = rev ? t1 - 1 - k : t0 + k;
      const int s = k % kStages;
      const uint32_t ph = static_cast<uint32_t>(k / kStages) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) break;
      body(t, base + static_cast<uint32_t>(s * kTileBytes));
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
  }
};

// Pass 1: colmax[n] = bits of max |dY*sx[m]|, colsum[n] += sum dY (float32
// within a block's rows, float64 across blocks), and with ROWMAX
// rowmax[m] = bits of max |dY*sw[n]| (one atomic per row per column block).
template <typename InT, bool ROWMAX>
__global__ void __launch_bounds__(kThreads) colstats_tma_kernel(
    const __grid_constant__ CUtensorMap tm, int64_t M, int N, const float* __restrict__ sx,
    uint32_t* __restrict__ colmax, double* __restrict__ colsum, const float* __restrict__ sw,
    uint32_t* __restrict__ rowmax, int32_t* __restrict__ status, int tiles_per_cta) {
  using T = Tile<InT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* buf = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t s_full[kStages], s_empty[kStages];
  __shared__ volatile int s_abort;
  // The final per-column reduction reuses the (drained) ring buffer.
  uint32_t(*s_max)[kCols] = reinterpret_cast<uint32_t(*)[kCols]>(buf);
  float(*s_sum)[kCols] = reinterpret_cast<float(*)[kCols]>(buf + 8 * kCols * 4);
  static_assert(8 * kCols * 8 <= kStages * kTileBytes, "reduction fits in the ring");
  Ring ring{buf, s_full, s_empty, &s_abort};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  ring.init(tid);
  __syncthreads();
  griddep_wait();  // dY and the factors (earlier kernels' outputs) are visible from here
  const int cb = blockIdx.x;
  const int tiles = static_cast<int>((M + T::kRows - 1) / T::kRows);
  const int t0 = blockIdx.y * tiles_per_cta;
  const int t1 = t0 + tiles_per_cta < tiles ? t0 + tiles_per_cta : tiles;
  const int nsub = min(kSub, (N - cb * kBlockCols + kCols - 1) / kCols);
  const int sub = warp % kSub;                      // this warp's quarter
  const bool live = warp < 8 && sub < nsub;         // it holds columns of the matrix
  const int col = cb * kBlockCols + sub * kCols + lane * 8;
  // Maxima as floats with NaN-propagating max (max.NaN.f32) over |x|
  // operands: a NaN or infinite product dY*s_x (an infinite dY in a row whose
  // s_x is 0 gives NaN) makes its column maximum NaN or +inf, and likewise
  // dY*s_w for the row maxima, which is exactly when the layer's definition
  // reports a non-finite value.  The column sums only feed db.
  float mx[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float sm[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint32_t rbad = 0;
  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_desc(&tm);
      ring.produce(&tm, cb, nsub, t0, t1, T::kRows);
    }
    __syncwarp();
  } else {
    float w8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (ROWMAX && col < N) load8(sw + col, w8);
    const uint32_t qoff = static_cast<uint32_t>(sub * (kTileBytes / kSub));
    // Lane j < kRowsPerWarp holds the factor s_x of row j of this warp's rows;
    // the next tile's are loaded while this one is worked on.
    constexpr int RW = T::kRowsPerWarp;
    const int rw0 = (warp / kSub) * RW;  // this warp's first row of a tile
    auto load_scale = [&](int t) {
      const int64_t m = static_cast<int64_t>(t) * T::kRows + rw0 + lane;
      return (lane < RW && t < t1 && m < M) ? __ldg(sx + m) : 0.0f;
    };
    float fcur = load_scale(t0);
    ring.consume(t0, t1, lane, [&](int t, uint32_t stage) {
      if (!live) return;  // a quarter past the last column: nothing loaded
      const uint32_t tile = stage + qoff;
      const float fnext = load_scale(t + 1);
      const int64_t m0 = static_cast<int64_t>(t) * T::kRows + rw0;
      uint32_t rmax = 0;  // lane j: the maximum of row j of this warp's rows
      // Two rows per step, so one three-operand max covers both.  Rows of
      // the tile past M were zero-filled by the copy and their factors are
      // 0: they add nothing to the column maxima and sums.
#pragma unroll
      for (int j = 0; j < RW; j += 2) {
        const int r = rw0 + j;
        float d0[8], d1[8];
        smem_load8<InT>(tile + (r * kCols + lane * 8) * sizeof(InT), d0);
        smem_load8<InT>(tile + ((r + 1) * kCols + lane * 8) * sizeof(InT), d1);
        const float f0 = __shfl_sync(0xFFFFFFFFu, fcur, j);
        const float f1 = __shfl_sync(0xFFFFFFFFu, fcur, j + 1);
        float rb0 = 0.0f, rb1 = 0.0f;
        // Products (only their magnitudes are used, no sum follows them) and
        // column sums two columns per instruction.
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const float2 a = make_float2(d0[i], d0[i + 1]), b = make_float2(d1[i], d1[i + 1]);
          const float2 pa = mul2(a, make_float2(f0, f0)), pb = mul2(b, make_float2(f1, f1));
          mx[i] = fmax3_nan(mx[i], fabsf(pa.x), fabsf(pb.x));
          mx[i + 1] = fmax3_nan(mx[i + 1], fabsf(pa.y), fabsf(pb.y));
          const float2 ss = add2(add2(make_float2(sm[i], sm[i + 1]), a), b);
          sm[i] = ss.x;
          sm[i + 1] = ss.y;
          if (ROWMAX) {
            const float2 wv = make_float2(w8[i], w8[i + 1]);
            const float2 ra = mul2(a, wv), rv = mul2(b, wv);
            rb0 = fmax3_nan(rb0, fabsf(ra.x), fabsf(ra.y));
            rb1 = fmax3_nan(rb1, fabsf(rv.x), fabsf(rv.y));
          }
        }
        if (ROWMAX) {
          // Non-negative floats order like their bit patterns; NaN sorts last.
          const uint32_t u0 = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(rb0));
          const uint32_t u1 = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(rb1));
          rmax = lane == j ? u0 : (lane == j + 1 ? u1 : rmax);
        }
      }
      if (ROWMAX && lane < RW && m0 + lane < M) {
        atomicMax(rowmax + m0 + lane, rmax);
        rbad = max(rbad, rmax);
      }
      fcur = fnext;
    });
  }
  griddep_launch_dependents();
  __syncthreads();  // ring drained (the producer waited for its copies): reuse it
  if (warp < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s_max[warp][i * 32 + lane] = __float_as_uint(mx[i]);  // column lane*8+i at slot i*32+lane
      s_sum[warp][i * 32 + lane] = sm[i];
    }
  }
  __syncthreads();
  for (int c = tid; c < kBlockCols; c += blockDim.x) {
    if (cb * kBlockCols + c >= N) break;
    const int q = c / kCols, j = c % kCols;
    const int slot = (j % 8) * 32 + j / 8;
    uint32_t a = 0;
    double t = 0.0;
#pragma unroll
    for (int h = 0; h < 8 / kSub; ++h) {  // the warps of quarter q
      a = max(a, s_max[q + kSub * h][slot]);
      t += static_cast<double>(s_sum[q + kSub * h][slot]);
    }
    // A NaN or infinite maximum: report it (the affected outputs are
    // unspecified).
    if (a >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
    atomicMax(colmax + cb * kBlockCols + c, a);
    atomicAdd(colsum + cb * kBlockCols + c, t);
  }
  if (ROWMAX && rbad >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
  if (tid == 0 && s_abort) atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

// 127/amax and amax/127 of a maximum kept as float bits (0 for a zero maximum).
__device__ __forceinline__ float inv_of(uint32_t bits) {
  const float amax = __uint_as_float(bits);
  return amax == 0.0f ? 0.0f : 127.0f / amax;
}
__device__ __forceinline__ float scale_of(uint32_t bits) {
  const float amax = __uint_as_float(bits);
  return amax == 0.0f ? 0.0f : amax / 127.0f;
}

// Pass 2: q2[m,n] = rne((dY*rs2[m]) * cinv2[n]) and, with Q1,
// q1[m,n] = rne((dY*cs1[n]) * rinv1[m]), where cinv2 = 127/colmax and
// rinv1 = 127/rowmax come straight from pass 1's maxima (IEEE divisions, a
// few per CTA and tile).  The scales the GEMM epilogues need are written
// here too, each by one CTA: s2 = colmax/127 and db (the column sums) by
// the first row group, s1 = rowmax/127 by the first column block.  Each CTA
// walks its tiles in the reverse of pass 1's order, so it starts on the
// tiles pass 1 read last, which are the likeliest to be still in L2.
template <typename InT, bool Q1>
__global__ void __launch_bounds__(kThreads) dualquant_tma_kernel(
    const __grid_constant__ CUtensorMap tm, int64_t M, int N, const float* __restrict__ cs1,
    const float* __restrict__ rs2, const uint32_t* __restrict__ colmax,
    const double* __restrict__ colsum, const uint32_t* __restrict__ rowmax,
    float* __restrict__ s1, float* __restrict__ s2, float* __restrict__ db,
    int8_t* __restrict__ q1, int8_t* __restrict__ q2, int32_t* __restrict__ status,
    int tiles_per_cta) {
  using T = Tile<InT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* buf = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t s_full[kStages], s_empty[kStages];
  __shared__ volatile int s_abort;
  Ring ring{buf, s_full, s_empty, &s_abort};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  ring.init(tid);
  __syncthreads();
  griddep_wait();  // dY and the maxima (earlier kernels' outputs) are visible from here
  const int cb = blockIdx.x;
  const int tiles = static_cast<int>((M + T::kRows - 1) / T::kRows);
  const int t0 = blockIdx.y * tiles_per_cta;
  const int t1 = t0 + tiles_per_cta < tiles ? t0 + tiles_per_cta : tiles;
  const int nsub = min(kSub, (N - cb * kBlockCols + kCols - 1) / kCols);
  const int sub = warp % kSub;                      // this warp's quarter
  const bool live = warp < 8 && sub < nsub;         // it holds columns of the matrix
  const int col = cb * kBlockCols + sub * kCols + lane * 8;
  const bool cv = col < N;
  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_desc(&tm);
      ring.produce(&tm, cb, nsub, t0, t1, T::kRows, true);
    }
    __syncwarp();
  } else {
    float w8[8] = {0, 0, 0, 0, 0, 0, 0, 0}, iv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (cv) {
      const uint4 c0 = __ldg(reinterpret_cast<const uint4*>(colmax + col));
      const uint4 c1 = __ldg(reinterpret_cast<const uint4*>(colmax + col + 4));
      const uint32_t cm[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) iv[i] = inv_of(cm[i]);
      if (blockIdx.y == 0 && warp < kSub) {  // one writer per column
        float sc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sc[i] = scale_of(cm[i]);
        reinterpret_cast<float4*>(s2 + col)[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
        reinterpret_cast<float4*>(s2 + col)[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
        if (db) {
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = static_cast<float>(colsum[col + i]);
          reinterpret_cast<float4*>(db + col)[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
          reinterpret_cast<float4*>(db + col)[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
        }
      }
      if (Q1) load8(cs1 + col, w8);
    }
    // Lane j < kRowsPerWarp holds the factors of row j of this warp's rows;
    // the next tile's are loaded while this one is worked on.
    constexpr int RW = T::kRowsPerWarp;
    const int rw0 = (warp / kSub) * RW;  // this warp's first row of a tile
    const uint32_t qoff = static_cast<uint32_t>(sub * (kTileBytes / kSub));
    auto load_rows = [&](int t, float& f2, float& r1) {
      const int64_t m = static_cast<int64_t>(t) * T::kRows + rw0 + lane;
      const bool in = lane < RW && t >= t0 && t < t1 && m < M;
      f2 = in ? __ldg(rs2 + m) : 0.0f;
      r1 = 0.0f;
      if (Q1 && in) {
        const uint32_t rb = __ldg(rowmax + m);
        r1 = inv_of(rb);
        if (cb == 0 && sub == 0) s1[m] = scale_of(rb);  // one writer per row
      }
    };
    float f2cur, r1cur;
    load_rows(t1 - 1, f2cur, r1cur);
    ring.consume(t0, t1, lane, [&](int t, uint32_t stage) {
      if (!live) return;  // a quarter past the last column: nothing loaded
      const uint32_t tile = stage + qoff;
      float f2next, r1next;
      load_rows(t - 1, f2next, r1next);
#pragma unroll
      for (int j = 0; j < RW; ++j) {
        const int r = rw0 + j;
        const int64_t m = static_cast<int64_t>(t) * T::kRows + r;
        const float f2 = __shfl_sync(0xFFFFFFFFu, f2cur, j);
        const float r1 = Q1 ? __shfl_sync(0xFFFFFFFFu, r1cur, j) : 0.0f;
        if (m < M && cv) {
          float d[8];
          smem_load8<InT>(tile + (r * kCols + lane * 8) * sizeof(InT), d);
          // Products two at a time; the rounding add one at a time (a packed
          // multiply whose result feeds a packed add is fused into one fma by
          // the code generator, which would skip the product's rounding).
          uint32_t b[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 v = mul2(mul2(make_float2(d[i], d[i + 1]), make_float2(f2, f2)),
                                  make_float2(iv[i], iv[i + 1]));
            b[i] = __float_as_uint(__fadd_rn(v.x, kRneMagic));
            b[i + 1] = __float_as_uint(__fadd_rn(v.y, kRneMagic));
          }
          *reinterpret_cast<uint2*>(q2 + m * N + col) =
              make_uint2(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]));
          if (Q1) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const float2 v = mul2(mul2(make_float2(d[i], d[i + 1]), make_float2(w8[i], w8[i + 1])),
                                    make_float2(r1, r1));
              b[i] = __float_as_uint(__fadd_rn(v.x, kRneMagic));
              b[i + 1] = __float_as_uint(__fadd_rn(v.y, kRneMagic));
            }
            *reinterpret_cast<uint2*>(q1 + m * N + col) =
                make_uint2(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]));
          }
        }
      }
      f2cur = f2next;
      r1cur = r1next;
    }, true);
  }
  griddep_launch_dependents();
  __syncthreads();
  if (tid == 0 && s_abort) atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

constexpr int kSmemBytes = 1024 + kStages * kTileBytes;

struct Grid {
  dim3 grid;
  int tiles_per_cta;
};

// Column blocks x row groups, about `per_sm` resident CTAs per SM in total.
Grid plan(int64_t M, int64_t N, int rows_per_tile, int per_sm) {
  const int cbs = static_cast<int>((N + kBlockCols - 1) / kBlockCols);
  const int tiles = static_cast<int>((M + rows_per_tile - 1) / rows_per_tile);
  int groups = device_info().sms * per_sm / cbs;  // round down: one wave of resident CTAs
  if (groups > tiles) groups = tiles;
  if (groups < 1) groups = 1;
  const int per = (tiles + groups - 1) / groups;
  groups = (tiles + per - 1) / per;
  return {dim3(static_cast<unsigned>(cbs), static_cast<unsigned>(groups)), per};
}

// Opt kernel K in to kSmemBytes of dynamic shared memory, once per device
// (one flag set per kernel: the template is keyed on the kernel itself).
template <auto K>
void allow_smem() {
  static bool done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !__atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) {
    cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    __atomic_store_n(&done[dev], true, __ATOMIC_RELEASE);
  }
}

template <typename InT>
bool dy_map(CUtensorMap* tm, const void* dy, int64_t M, int64_t N) {
  return encode_tmap_2d(tm, sizeof(InT), dy, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                        static_cast<uint64_t>(N) * sizeof(InT), kCols, Tile<InT>::kRows, false);
}

template <typename InT>
cudaError_t colstats_t(const void* dy, int64_t M, int64_t N, const float* sx, uint32_t* colmax,
                       double* colsum, const float* sw, uint32_t* rowmax, int32_t* status,
                       cudaStream_t s) {
  CUtensorMap tm;
  if (!dy_map<InT>(&tm, dy, M, N)) return cudaErrorInvalidValue;
  const Grid g = plan(M, N, Tile<InT>::kRows, 2);
  cudaError_t e = cudaSuccess;
  if (rowmax) {
    allow_smem<colstats_tma_kernel<InT, true>>();
    e = launch_pdl(colstats_tma_kernel<InT, true>, g.grid, dim3(kThreads), kSmemBytes, s, tm, M,
                   static_cast<int>(N), sx, colmax, colsum, sw, rowmax, status, g.tiles_per_cta);
  } else {
    allow_smem<colstats_tma_kernel<InT, false>>();
    e = launch_pdl(colstats_tma_kernel<InT, false>, g.grid, dim3(kThreads), kSmemBytes, s, tm, M,
                   static_cast<int>(N), sx, colmax, colsum, sw, rowmax, status, g.tiles_per_cta);
  }
  count_launches(1);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <typename InT>
cudaError_t dualquant_t(const void* dy, int64_t M, int64_t N, const float* cs1, const float* rs2,
                        const uint32_t* colmax, const double* colsum, const uint32_t* rowmax,
                        float* s1, float* s2, float* db, int8_t* q1, int8_t* q2,
                        int32_t* status, cudaStream_t s) {
  CUtensorMap tm;
  if (!dy_map<InT>(&tm, dy, M, N)) return cudaErrorInvalidValue;
  const Grid g = plan(M, N, Tile<InT>::kRows, 2);
  cudaError_t e = cudaSuccess;
  if (q1) {
    allow_smem<dualquant_tma_kernel<InT, true>>();
    e = launch_pdl(dualquant_tma_kernel<InT, true>, g.grid, dim3(kThreads), kSmemBytes, s, tm, M,
                   static_cast<int>(N), cs1, rs2, colmax, colsum, rowmax, s1, s2, db, q1, q2,
                   status, g.tiles_per_cta);
  } else {
    allow_smem<dualquant_tma_kernel<InT, false>>();
    e = launch_pdl(dualquant_tma_kernel<InT, false>, g.grid, dim3(kThreads), kSmemBytes, s, tm, M,
                   static_cast<int>(N), cs1, rs2, colmax, colsum, rowmax, s1, s2, db, q1, q2,
                   status, g.tiles_per_cta);
  }
  count_launches(1);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace

cudaError_t launch_colstats(const void* dy, int dyt, int64_t M, int64_t N, const float* sx,
                            uint32_t* colmax, double* colsum, const float* sw, uint32_t* rowmax,
                            int32_t* status, cudaStream_t s) {
  if (dyt == QL_BF16)
    return colstats_t<__nv_bfloat16>(dy, M, N, sx, colmax, colsum, sw, rowmax, status, s);
  return colstats_t<float>(dy, M, N, sx, colmax, colsum, sw, rowmax, status, s);
}

cudaError_t launch_dualquant(const void* dy, int dyt, int64_t M, int64_t N, const float* cs1,
                             const float* rs2, const uint32_t* colmax, const double* colsum,
                             const uint32_t* rowmax, float* s1, float* s2, float* db, int8_t* q1,
                             int8_t* q2, int32_t* status, cudaStream_t s) {
  if (dyt == QL_BF16)
    return dualquant_t<__nv_bfloat16>(dy, M, N, cs1, rs2, colmax, colsum, rowmax, s1, s2, db, q1,
                                      q2, status, s);
  return dualquant_t<float>(dy, M, N, cs1, rs2, colmax, colsum, rowmax, s1, s2, db, q1, q2,
                            status, s);
}

}  // namespace ql
