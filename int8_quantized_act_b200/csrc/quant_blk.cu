// quant_blk.cu - per-row int8 quantization of bf16 rows, optionally rotated
// by a block-Hadamard of width <= 128, with two threads per 128-column block
// of a row (OneTrainer PR #1681 "Int8 conv rot", commit note item 1: the
// activations are quantized per row on every call, after the rotation of the
// opening summary).
//
// The thread with half bit hb holds columns 64*hb .. 64*hb+63 of its block
// in registers as 32 pairs (column j, column j + 32) of the half, so the
// butterflies h = 1..16 act on both quarters with one packed f32x2 addition
// or subtraction and h = 32 (the pair's own two values) is scalar; h = 64
// pairs the two halves with one shuffle per pair (the pairs of the upper
// half are held swapped, so both halves send the same component).
// The row maximum is a three-operand NaN-propagating max.  About 110
// registers a thread, so a 256-thread CTA (R rows of a tile) runs twice per
// SM, 16 warps: enough to hide the latency that 8 warps of a
// thread-per-block layout left exposed.  Rows reach shared memory by TMA, a
// ring of tiles per CTA; a thread reads its own 128-byte line of the tile,
// and the copy's 128-byte swizzle puts the 8 threads of a load phase on
// distinct banks.  The codes leave through two swizzled shared-memory tiles
// in turn, one TMA store per tile issued while the next tile is rotated, so
// every global write is a whole line (16-byte stores from registers, which
// leave each 32-byte sector half written per instruction, measured slower).
#include <algorithm>

#include "launch.h"
#include "rowops.cuh"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

constexpr int kBlkThreads = 256;     // 2 * R * (cols / 128) <= 256
constexpr int kBlkMaxRows = 32;      // rows per tile
constexpr int kBlkStagesMax = 4;

// The butterflies of fwht_block for blocks of HB (0 = none, 2..128) columns
// on the layout above, in the same order h = 1, 2, ..., HB/2 and with the
// same IEEE operations, then one multiply by c.  For HB = 128 the upper half
// (hb = 1) holds its pairs swapped, (column 32 + j, column j) of the half, so
// that h = 64 needs one shuffle a pair: both halves send their y value.
// h = 32 then forms lower + upper and lower - upper as fma(+-1, ., .), exact
// like the addition; after h = 64 the lower half holds (column j, column
// 64 + j) of the block and the upper half (column 32 + j, -(column 96 + j)),
// the sign put right by the multiply by c.
template <int HB>
__device__ __forceinline__ void fwht_half(float2 (&p)[32], int hb, float c) {
#pragma unroll
  for (int h = 1; h < 32 && h < HB; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const float2 a = p[i], b = p[i + h];
        p[i] = add2(a, b);
        p[i + h] = sub2(a, b);
      }
    }
  }
  if constexpr (HB == 64) {  // h = 32: the pair's own two values
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float a = p[i].x, b = p[i].y;
      p[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
  }
  if constexpr (HB == 128) {
    const float sg = hb ? -1.0f : 1.0f;
    // h = 32 on (lower, upper) = (x, y), or (y, x) in the upper half
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float x = p[i].x, y = p[i].y;
      p[i] = make_float2(__fmaf_rn(sg, x, y), __fmaf_rn(-sg, y, x));
    }
    // h = 64: the lower half pairs its x with the upper half's y, the upper
    // half its x with the lower half's y
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float x = p[i].x;
      const float r = __shfl_xor_sync(0xFFFFFFFFu, p[i].y, 1);
      p[i] = make_float2(__fadd_rn(x, r), __fsub_rn(x, r));
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], make_float2(c, sg * c));
  } else if constexpr (HB > 0) {
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], make_float2(c, c));
  }
}

// Codes of 16 values (component Y of the pairs m[i0..i0+15], each already
// the rounded product v * inv) as one 16-byte word: rne through the adder.
// The products are formed two at a time (mul.rn.f32x2) and the additions
// one at a time: a packed multiply followed by a packed add of its result
// is fused into one packed fma by the code generator (seen on sm_100a
// with -fmad=false), which would skip the rounding of the product.
template <bool Y>
__device__ __forceinline__ uint4 codes16(const float2 (&m)[32], int i0) {
  uint32_t b[16];
#pragma unroll
  for (int k = 0; k < 16; ++k)
    b[k] = __float_as_uint(__fadd_rn(Y ? m[i0 + k].y : m[i0 + k].x, kRneMagic));
  return make_uint4(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]),
                    pack_codes(b[8], b[9], b[10], b[11]), pack_codes(b[12], b[13], b[14], b[15]));
}

// tm_x: bf16 rows as [rows][cols / 64][64] (a 128-column block = two
// 128-byte lines), box = R rows, 128-byte swizzle.  tm_q: codes as
// [rows][cols / 128][128], box = R rows, 128-byte swizzle.  Thread t holds
// half t & 1 of block (t >> 1) % nb of tile row (t >> 1) / nb.  One barrier a
// tile: after it the row maxima are complete, every thread has read the
// tile's stage (thread 0 refills it), the codes of the previous tile are in
// their code tile (thread 0 stores them), and the maxima of the tile before
// last are no longer read (their slot is cleared for the tile after next).
// Bounded waits: on a time-out the CTA reports QL_ERR_TIMEOUT, lets its
// copies land and returns.
template <int HB>
__global__ void __launch_bounds__(kBlkThreads, 2) quant_blk_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
    int64_t rows, int nb, int R, float hc, unsigned flags, float* __restrict__ row_scale,
    int32_t* __restrict__ status, int stages, int stage_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* out = smem + stages * stage_bytes;
  __shared__ uint32_t s_rmax[3][kBlkMaxRows];
  __shared__ __align__(8) uint64_t s_full[kBlkStagesMax];
  __shared__ volatile int s_abort;
  const int t = threadIdx.x;
  const int hb = t & 1;                  // half of the block
  const int blk = t >> 1;                // block of the tile
  const int rl = blk / nb;               // row of the tile
  const int b = blk - rl * nb;           // 128-column block of the row
  const bool active = rl < R;
  const int64_t tiles = (rows + R - 1) / R;
  const int64_t mine = tiles > blockIdx.x ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const uint32_t tile_bytes = static_cast<uint32_t>(R) * static_cast<uint32_t>(nb) * 256u;
  if (t == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(smem_u32(&s_full[s]), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (t < 2 * kBlkMaxRows) s_rmax[t / kBlkMaxRows][t % kBlkMaxRows] = 0u;
  __syncthreads();
  griddep_wait();  // the rows (a previous kernel's output) are visible from here
  if (t == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_q);
    for (int s = 0; s < stages && s < mine; ++s) {
      const int64_t tile = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
      mbar_arrive_expect_tx(smem_u32(&s_full[s]), tile_bytes);
      tma_load_3d(smem_u32(smem + s * stage_bytes), &tm_x, smem_u32(&s_full[s]), 0, 0,
                  static_cast<int>(tile * R));
    }
  }
  const int tl = active ? t : 0;    // the line of a stage this thread reads
  const int key = tl & 7;           // its swizzle key
  // 16-byte pieces of the line that hold the x and y columns of the pairs
  // (swapped in the upper half of a 128-column block).
  const int xo = (HB == 128 && hb) ? 4 : 0, yo = 4 - xo;
  // 16-byte pieces of the block's 128 codes that receive them.
  const int cx = HB == 128 ? 2 * hb : 4 * hb;
  const int cy = HB == 128 ? 4 + 2 * hb : 4 * hb + 2;
  const int okey = blk & 7;
  const uint32_t out_bytes = static_cast<uint32_t>(R) * static_cast<uint32_t>(nb) * 128u;
  const uint32_t out_stride = (out_bytes + 1023u) & ~1023u;
  int64_t done = 0;
  for (int64_t i = 0; i < mine; ++i) {
    const int st = static_cast<int>(i % stages);
    const uint32_t parity = static_cast<uint32_t>((i / stages) & 1);
    const int64_t tile = blockIdx.x + i * gridDim.x;
    const int64_t r = tile * R + rl;
    const int slot = static_cast<int>(i % 3);
    // A thread that gives up (mbar_wait raises s_abort) still takes part in
    // the barrier below; the CTA leaves the loop together after it.  It reads
    // the stage regardless (in bounds; the values are not used), as does a
    // thread past the tile's rows (line 0; its values go nowhere).
    (void)mbar_wait(smem_u32(&s_full[st]), parity, &s_abort);
    float2 p[32];
    {
      const uint32_t line = smem_u32(smem) + st * stage_bytes + tl * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 u = lds128(line + (((c + xo) ^ key) << 4));  // cols xo*8 + 8c..
        const uint4 w = lds128(line + (((c + yo) ^ key) << 4));  // cols yo*8 + 8c..
        const uint32_t a4[4] = {u.x, u.y, u.z, u.w}, b4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          p[8 * c + 2 * e] = make_float2(__uint_as_float(a4[e] << 16), __uint_as_float(b4[e] << 16));
          p[8 * c + 2 * e + 1] = make_float2(__uint_as_float(a4[e] & 0xFFFF0000u),
                                             __uint_as_float(b4[e] & 0xFFFF0000u));
        }
      }
    }
    fwht_half<HB>(p, hb, hc);
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      m0 = fmax3_nan(m0, fabsf(p[j].x), fabsf(p[j].y));
      m1 = fmax3_nan(m1, fabsf(p[j + 1].x), fabsf(p[j + 1].y));
    }
    float m = fmax_nan(m0, m1);
    m = fmax_nan(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));  // the block's two halves
    // Non-negative floats order like their bit patterns; NaN sorts last.
    if (active && hb == 0) atomicMax(&s_rmax[slot][rl], __float_as_uint(m));
    if (t == 0) bulk_wait_read_all();  // the store two tiles back has read code tile i & 1
    __syncthreads();
    if (t == 0) {
      if (i > 0) {
        tma_store_3d(&tm_q, smem_u32(out) + ((i - 1) & 1) * out_stride, 0, 0,
                     static_cast<int>((tile - gridDim.x) * R));
        bulk_commit();
      }
      if (i + stages < mine && !s_abort) {
        fence_proxy_async_smem();
        const int64_t tn = blockIdx.x + (i + stages) * gridDim.x;
        mbar_arrive_expect_tx(smem_u32(&s_full[st]), tile_bytes);
        tma_load_3d(smem_u32(smem + st * stage_bytes), &tm_x, smem_u32(&s_full[st]), 0, 0,
                    static_cast<int>(tn * R));
      }
      const int nxt = static_cast<int>((i + 2) % 3);  // the tile after next
      for (int k = 0; k < R; ++k) s_rmax[nxt][k] = 0u;
    }
    if (s_abort) break;
    const uint32_t mb = s_rmax[slot][rl < R ? rl : 0];
    const float amax = __uint_as_float(mb);
    const float inv = mb == 0 ? 0.0f : 127.0f / amax;
    if (active) {
      const uint32_t ol = smem_u32(out) + (i & 1) * out_stride + blk * 128;
#pragma unroll
      for (int j = 0; j < 32; ++j) p[j] = mul2(p[j], make_float2(inv, inv));
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        sts128(ol + (((cx + u) ^ okey) << 4), codes16<false>(p, 16 * u));
        sts128(ol + (((cy + u) ^ okey) << 4), codes16<true>(p, 16 * u));
      }
    }
    if (active && r < rows) {
      if (b == 0 && hb == 0) {
        row_scale[r] = mb == 0 ? 0.0f : amax / 127.0f;
        if (mb == 0 && (flags & QL_REJECT_ZERO_ROWS)) atomicOr(status, 1 << QL_ERR_ZERO_ROW);
        if (mb >= kInfBits) atomicOr(status, 1 << QL_ERR_NONFINITE);
      }
    }
    fence_proxy_async_smem();  // the codes, before a store reads them
    done = i + 1;
  }
  griddep_launch_dependents();
  __syncthreads();
  if (t == 0 && !s_abort && mine > 0) {
    const int64_t last = blockIdx.x + (mine - 1) * gridDim.x;
    tma_store_3d(&tm_q, smem_u32(out) + ((mine - 1) & 1) * out_stride, 0, 0,
                 static_cast<int>(last * R));
    bulk_commit();
  }
  if (t == 0 && s_abort) {
    // Timed out: let every load already issued (tiles done .. done+stages-1)
    // land before the CTA exits.
    atomicOr(status, 1 << QL_ERR_TIMEOUT);
    for (int64_t i = done; i < mine && i < done + stages; ++i)
      mbar_wait_drain(smem_u32(&s_full[i % stages]), static_cast<uint32_t>((i / stages) & 1));
  }
  if (t == 0) bulk_wait_all();
}

template <int HB>
cudaError_t launch_blk_t(const CUtensorMap& tx, const CUtensorMap& tq, int64_t rows, int nb,
                         int R, int threads, float hc, unsigned flags, float* rs, int32_t* st,
                         int stage_bytes, int out_bytes, cudaStream_t s) {
  auto kern = quant_blk_kernel<HB>;
  // Opt in to the largest dynamic shared memory the kernel can take beside
  // its static arrays, once per device (0: not yet).
  static int static_bytes[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int static_smem = dev < 64 ? __atomic_load_n(&static_bytes[dev], __ATOMIC_ACQUIRE) : 0;
  if (static_smem == 0) {
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               device_info().smem_optin - static_cast<int>(fa.sharedSizeBytes));
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return e;
    }
    static_smem = std::max(1, static_cast<int>(fa.sharedSizeBytes));
    if (dev < 64) __atomic_store_n(&static_bytes[dev], static_smem, __ATOMIC_RELEASE);
  }
  // Two CTAs per SM with the deepest ring that fits (at least two stages);
  // shared memory per SM is 228 KB with 1 KB reserved per CTA.
  int per_sm = 2, stages = 0;
  for (; per_sm >= 1; --per_sm) {
    const int budget = std::min(device_info().smem_optin, 233472 / per_sm - 1024) - static_smem -
                       1024 /* alignment slack of the dynamic buffer */ - 2 * out_bytes;
    stages = std::min(kBlkStagesMax, budget / stage_bytes);
    if (stages >= 2) break;
  }
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const int smem = 1024 + stages * stage_bytes + 2 * out_bytes;
  const int64_t tiles = (rows + R - 1) / R;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, static_cast<int64_t>(device_info().sms) * per_sm));
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(threads), static_cast<size_t>(smem), s, tx,
                                   tq, rows, nb, R, hc, flags, rs, st, stages, stage_bytes);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace

bool quant_blk_eligible(int64_t rows, int64_t cols, int64_t ldx, int B, bool col_scale) {
  if (col_scale) return false;
  if (cols % 128 != 0 || cols < 128 || cols > 128 * (kBlkThreads / 2) || B > 128) return false;
  if ((ldx * 2) % 16 != 0 || rows > INT32_MAX) return false;
  const int nb = static_cast<int>(cols / 128);
  const int R = std::min(kBlkMaxRows, (kBlkThreads / 2) / nb);
  // At least one tile per SM; fewer rows go to the register kernels.
  return rows >= static_cast<int64_t>(R) * device_info().sms;
}

cudaError_t launch_quant_blk(const void* x, int64_t rows, int64_t cols, int64_t ldx, int B,
                             float hc, unsigned flags, int8_t* q, int64_t ldq, float* rs,
                             int32_t* st, cudaStream_t s) {
  const int nb = static_cast<int>(cols / 128);
  const int R = std::min(kBlkMaxRows, (kBlkThreads / 2) / nb);
  const int threads = (2 * R * nb + 31) / 32 * 32;
  CUtensorMap tx, tq;
  if (!encode_rows_128b(&tx, 2, x, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                        static_cast<uint64_t>(ldx) * 2, static_cast<uint32_t>(R)))
    return cudaErrorInvalidValue;
  {
    const uint64_t dims[3] = {128, static_cast<uint64_t>(nb), static_cast<uint64_t>(rows)};
    const uint64_t strides[2] = {128, static_cast<uint64_t>(ldq)};
    const uint32_t box[3] = {128, static_cast<uint32_t>(nb), static_cast<uint32_t>(R)};
    if (!encode_tmap(&tq, 1, q, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  const int stage_bytes = (R * nb * 256 + 1023) / 1024 * 1024;
  const int out_bytes = (R * nb * 128 + 1023) / 1024 * 1024;
  cudaError_t e = cudaErrorInvalidValue;
#define QL_BLK(HB) \
  e = launch_blk_t<HB>(tx, tq, rows, nb, R, threads, hc, flags, rs, st, stage_bytes, out_bytes, s)
  switch (B) {
    case 0: QL_BLK(0); break;
    case 2: QL_BLK(2); break;
    case 4: QL_BLK(4); break;
    case 8: QL_BLK(8); break;
    case 16: QL_BLK(16); break;
    case 32: QL_BLK(32); break;
    case 64: QL_BLK(64); break;
    case 128: QL_BLK(128); break;
    default: break;
  }
#undef QL_BLK
  count_launches(1);
  return e;
}

}  // namespace ql
