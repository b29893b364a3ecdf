// gemm_i8.cu - int8 x int8 -> int32 GEMM on the sm_100a tensor cores
// (tcgen05.mma.kind::i8) with the layer's scale/bias epilogues.
//
// One kernel serves the three products of the layer (OneTrainer PR #1681
// uses torch._int_mm for the forward one):
//   forward  y  = X_q W_q^T      A = X_q   [M,K] K-major,  B = W_q [N,K] K-major
//   input    dX = dYq_r W_q      A = dYq_r [M,N] K-major,  B = W_q [N,K] MN-major
//   weight   dW = dYq_c^T X_q    A = dYq_c [M,N] MN-major, B = X_q [M,K] MN-major
// tcgen05 reads 8-bit operands in either major-ness, so no transposed copy
// of any operand is ever written.
//
// Structure (persistent, one CTA per SM, 6 warps):
//   warp 0      TMA producer: 128x128-byte A tile + 256x128-byte B tile per
//               stage into a 4-stage ring of 128B-swizzled shared memory.
//   warp 1      allocates 512 TMEM columns (two 128x256 int32 accumulators),
//               one elected thread issues tcgen05.mma (M=128, N=256, K=32)
//               and tcgen05.commit to release ring stages / hand accumulators
//               to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter, scale, bias,
//               optional in-register block-Hadamard, 128-bit global stores;
//               they drain one accumulator while the MMA fills the other.
// Tiles whose rows / columns / contraction run past the matrix are zero-
// filled by TMA, so M has no floor and tails need no special path.
// No TMA multicast is used anywhere.
#include <cuda.h>
#include <algorithm>
#include <type_traits>
#include <cuda_bf16.h>

#include "launch.h"
#include "sm100.cuh"
#include "../../include/qlinear.h"

namespace ql {

namespace {

constexpr int BM = 128;                // tile rows (TMEM lanes)
constexpr int BN = 256;                // tile columns (TMEM columns per accumulator)
constexpr int BK = 128;                // contraction bytes per stage (4 MMAs of K=32)
constexpr int STAGES = 4;
// Longest int32-safe contraction split in 128-element blocks: 1023 * 128 =
// 130,944 <= 131,071 = floor((2^31 - 1) / 128^2).
constexpr int64_t kMaxSplitBlocks = 1023;
// Most contraction splits used to spread a small (<= 128-row) output.
constexpr int64_t kMaxSmallSplits = QL_SMALL_OUTPUT_SPLITS;
constexpr int A_BYTES = BM * BK;       // 16 KiB
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;      // 512: the whole TMEM of the SM
// Float32 epilogues stage each warp's 32 x 32 chunk in shared memory (rows
// padded to 33 words) so that the stores go out as whole 128-byte row pieces.
constexpr int kEpiStageFloats = 32 * 33;
constexpr int kEpiStageBytes = 4 * 4 * kEpiStageFloats;  // 4 epilogue warps

// The single-CTA kernel's tile width: 256 columns, or 64 for outputs of one
// 128-row slab whose 256-wide tiles would leave most SMs idle (the forward at
// a few tokens streams the whole weight through few CTAs otherwise); the
// narrower tile takes twice the stages to keep as many bytes in flight.
template <int TBN>
struct Single {
  static constexpr int kBN = TBN;
  static constexpr int kStages = TBN == 256 ? STAGES : 8;
  static constexpr int kBBytes = TBN * BK;
  static constexpr int kStageBytes = A_BYTES + kBBytes;
  static constexpr int kTmemCols = 2 * TBN;  // two accumulators, a power of two >= 32
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 8 * kNumBars + 16 + kEpiStageBytes;
};

struct Epi {
  void* out;
  int64_t ldo;
  int64_t split_stride;  // elements between the outputs of successive contraction splits
  int rows, cols;
  const float* row_scale;
  const float* col_scale;
  const float* bias;
  float hc;
  // The Newton-Schulz steps in a bf16 kind::f16 epilogue (GemmEpilogue::ns_x,
  // ns_mirror); null / 0: none.
  const __nv_bfloat16* ns_x;
  __nv_bfloat16* ns_xt;
  int64_t ns_ldt;
  float ns_a, ns_c;
  int ns_mirror;
};

// Tile t of a tiles_m x tiles_n grid in grouped order: runs of `group`
// tile-rows are walked column by column, so the tiles in flight at any
// moment form a compact block and share their operand stripes in L2.
// group = 1 is plain row-major order (best when the B operand fits in L2 and
// every tile-row reuses it); the weight gradient, whose operands are both
// long stripes of the whole contraction, uses groups of 16.  group = 0 walks
// only the upper triangle (tm <= tn) of a square grid, row by row: the
// symmetric products X X^T and A A, whose lower tiles are the transposes.
__device__ __forceinline__ int tiles_per_split(int tiles_m, int tiles_n, int group) {
  return group == 0 ? tiles_m * (tiles_m + 1) / 2 : tiles_m * tiles_n;
}

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int group, int& tm,
                                            int& tn) {
  if (group == 0) {
    int r = t, m = 0;
    while (r >= tiles_m - m) {
      r -= tiles_m - m;
      ++m;
    }
    tm = m;
    tn = m + r;
    return;
  }
  const int per_group = group * tiles_n;
  const int g = t / per_group;
  const int first = g * group;
  const int rows = tiles_m - first < group ? tiles_m - first : group;
  const int r = t - g * per_group;
  tm = first + r % rows;
  tn = r / rows;
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N % 32 == 0, "chunks of 32 columns");
#pragma unroll
  for (int j = 0; j < N / 32; ++j)
    tmem_ld32(taddr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * j]));
}

// In-register block-Hadamard along one thread's row segment: blocks of HB
// consecutive values, butterflies h = 1..HB/2 in order, then times hc.
template <int N, int HB>
__device__ __forceinline__ void fwht_regs(float (&v)[N], float hc) {
#pragma unroll
  for (int h = 1; h < HB; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = v[i] * hc;
}

__device__ __forceinline__ void store16(float* p, const float* v) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* v) {
  reinterpret_cast<uint4*>(p)[0] =
      make_uint4(bf16x2(v[0], v[1]), bf16x2(v[2], v[3]), bf16x2(v[4], v[5]), bf16x2(v[6], v[7]));
  reinterpret_cast<uint4*>(p)[1] = make_uint4(bf16x2(v[8], v[9]), bf16x2(v[10], v[11]),
                                              bf16x2(v[12], v[13]), bf16x2(v[14], v[15]));
}

// Epilogue of one 128-row slab of an accumulator tile: rows row0 + 32*quarter
// + lane, columns col0 .. col0+255 of the output.  All 32 lanes of the warp
// must call it (tcgen05.ld is warp-collective); rows/columns past the output
// are computed but not stored.
template <typename OutT, int HB, bool F16, int TW = BN>
__device__ __forceinline__ void epilogue_tile(const Epi& ep, uint32_t acc_tmem, int quarter,
                                              int lane, int row0, int col0, float* stage) {
  constexpr int CH = HB > 32 ? HB : 32;  // columns per register chunk
  OutT* out = reinterpret_cast<OutT*>(ep.out);
  const int gr = row0 + quarter * 32 + lane;
  const bool row_ok = gr < ep.rows;

  const float rs = (row_ok && ep.row_scale) ? ep.row_scale[gr] : 1.0f;
  const uint32_t taddr = acc_tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
  for (int c0 = 0; c0 < TW; c0 += CH) {
    uint32_t r[CH];
    tmem_ld_cols<CH>(taddr + c0, r);
    tmem_wait_ld();
    const int gc0 = col0 + c0;
    float v[CH];
    if (row_ok && gc0 < ep.cols) {
#pragma unroll
      for (int i = 0; i < CH; ++i)
        v[i] = (F16 ? __uint_as_float(r[i]) : __int2float_rn(static_cast<int>(r[i]))) * rs;
      if (ep.col_scale || ep.bias) {
#pragma unroll
        for (int g = 0; g < CH / 16; ++g) {
          if (gc0 + 16 * g < ep.cols) {
            if (ep.col_scale) {
#pragma unroll
              for (int i = 0; i < 16; i += 4) {
                const float4 c4 = __ldg(reinterpret_cast<const float4*>(ep.col_scale + gc0 + 16 * g + i));
                v[16 * g + i] = v[16 * g + i] * c4.x;
                v[16 * g + i + 1] = v[16 * g + i + 1] * c4.y;
                v[16 * g + i + 2] = v[16 * g + i + 2] * c4.z;
                v[16 * g + i + 3] = v[16 * g + i + 3] * c4.w;
              }
            }
            if (ep.bias) {
#pragma unroll
              for (int i = 0; i < 16; i += 4) {
                const float4 b4 = __ldg(reinterpret_cast<const float4*>(ep.bias + gc0 + 16 * g + i));
                v[16 * g + i] = v[16 * g + i] + b4.x;
                v[16 * g + i + 1] = v[16 * g + i + 1] + b4.y;
                v[16 * g + i + 2] = v[16 * g + i + 2] + b4.z;
                v[16 * g + i + 3] = v[16 * g + i + 3] + b4.w;
              }
            }
          }
        }
      }
      if constexpr (HB > 0) fwht_regs<CH, HB>(v, ep.hc);
      if constexpr (F16 && HB == 0 && !std::is_same<OutT, float>::value) {
        // Newton-Schulz: x' = bf16(a*x + c*acc), x from the same position of X.
        if (ep.ns_x) {
          const __nv_bfloat16* xrow = ep.ns_x + static_cast<int64_t>(gr) * ep.ldo + gc0;
#pragma unroll
          for (int g = 0; g < CH / 16; ++g) {
            if (gc0 + 16 * g < ep.cols) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint4 u = *reinterpret_cast<const uint4*>(xrow + 16 * g + 8 * h);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  float* d = v + 16 * g + 8 * h + 2 * k;
                  d[0] = __fadd_rn(__fmul_rn(ep.ns_a, __uint_as_float(w[k] << 16)),
                                   __fmul_rn(ep.ns_c, d[0]));
                  d[1] = __fadd_rn(__fmul_rn(ep.ns_a, __uint_as_float(w[k] & 0xFFFF0000u)),
                                   __fmul_rn(ep.ns_c, d[1]));
                }
              }
            }
          }
        }
      }
      if constexpr (std::is_same<OutT, float>::value && HB == 0) {
        (void)0;
      } else {
        OutT* orow = out + static_cast<int64_t>(gr) * ep.ldo + gc0;
#pragma unroll
        for (int g = 0; g < CH / 16; ++g)
          if (gc0 + 16 * g < ep.cols) store16(orow + 16 * g, v + 16 * g);
      }
    }
    if constexpr (std::is_same<OutT, float>::value && HB == 0) {
      // Lane l holds row l of the warp's 32 rows; through the padded stage,
      // lane l then writes columns 4(l%8)..+3 of rows l/8, l/8+4, ...: each
      // store instruction covers four whole 128-byte row pieces.  (Every
      // lane takes part, whatever its row or column range.)
      if (gc0 < ep.cols) {
#pragma unroll
        for (int e = 0; e < 32; ++e) stage[lane * 33 + e] = row_ok ? v[e] : 0.0f;
        __syncwarp();
        const int cc = (lane & 7) * 4;
        const int rbase = row0 + quarter * 32;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + (lane >> 3);
          const float4 val = make_float4(stage[rr * 33 + cc], stage[rr * 33 + cc + 1],
                                         stage[rr * 33 + cc + 2], stage[rr * 33 + cc + 3]);
          if (rbase + rr < ep.rows && gc0 + cc < ep.cols)
            *reinterpret_cast<float4*>(out + static_cast<int64_t>(rbase + rr) * ep.ldo + gc0 + cc) = val;
        }
        __syncwarp();
      }
    }
    if constexpr (F16 && HB == 0 && !std::is_same<OutT, float>::value) {
      // The transposed copy of the stored values: into ns_xt, or with
      // ns_mirror (a symmetric product on its upper 256 x 256 tiles) into the
      // output's lower tile, for a strictly upper tile.  Through the padded
      // stage, lane l writes column gc0 + l of the chunk as a 64-byte piece of
      // row gc0 + l of the target (the chunk's valid rows only, a multiple of
      // 16).  Every lane takes part.
      const bool mirror = ep.ns_mirror && row0 / 256 < col0 / 256;
      __nv_bfloat16* tgt = mirror ? reinterpret_cast<__nv_bfloat16*>(ep.out) : ep.ns_xt;
      const int64_t ldt = mirror ? ep.ldo : ep.ns_ldt;
      if ((mirror || (ep.ns_x && ep.ns_xt)) && gc0 < ep.cols) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          stage[lane * 33 + e] = row_ok ? __bfloat162float(__float2bfloat16_rn(v[e])) : 0.0f;
        __syncwarp();
        const int rbase = row0 + quarter * 32;
        const int nrows = min(32, ep.rows - rbase);
        if (gc0 + lane < ep.cols && nrows > 0) {
          __nv_bfloat16* trow = tgt + static_cast<int64_t>(gc0 + lane) * ldt + rbase;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            if (8 * q8 < nrows) {
              uint32_t o[4];
#pragma unroll
              for (int k = 0; k < 4; ++k)
                o[k] = bf16x2(stage[(8 * q8 + 2 * k) * 33 + lane], stage[(8 * q8 + 2 * k + 1) * 33 + lane]);
              *reinterpret_cast<uint4*>(trow + 8 * q8) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        __syncwarp();
      }
    }
  }
}

// Raw int32 partial sums of one contraction split (no scaling), the same
// slab as epilogue_tile.
template <int TW = BN>
__device__ __forceinline__ void epilogue_tile_raw(const Epi& ep, uint32_t acc_tmem, int quarter,
                                                  int lane, int row0, int col0) {
  int32_t* out = reinterpret_cast<int32_t*>(ep.out);
  const int gr = row0 + quarter * 32 + lane;
  const bool row_ok = gr < ep.rows;
  const uint32_t taddr = acc_tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
  for (int c0 = 0; c0 < TW; c0 += 32) {
    uint32_t r[32];
    tmem_ld_cols<32>(taddr + c0, r);
    tmem_wait_ld();
    const int gc0 = col0 + c0;
    if (row_ok && gc0 < ep.cols) {
      int32_t* orow = out + static_cast<int64_t>(gr) * ep.ldo + gc0;
#pragma unroll
      for (int g = 0; g < 2; ++g)
        if (gc0 + 16 * g < ep.cols)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<uint4*>(orow + 16 * g)[i] =
                make_uint4(r[16 * g + 4 * i], r[16 * g + 4 * i + 1], r[16 * g + 4 * i + 2],
                           r[16 * g + 4 * i + 3]);
    }
  }
}

template <bool A_MN, bool B_MN, typename OutT, int HB, bool F16, int TBN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int tiles_m, int tiles_n, int kblocks, int kps, int group, int a_box_rows,
                   Epi ep, int32_t* status) {
  using C = Single<TBN>;
  static_assert(TBN == 256 || !B_MN, "narrow tiles read B K-major");
  constexpr int BN = C::kBN, STAGES = C::kStages, B_BYTES = C::kBBytes;
  constexpr int STAGE_BYTES = C::kStageBytes, TMEM_COLS = C::kTmemCols, NUM_BARS = C::kNumBars;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(tmem_slot + 4);  // scalar accesses only

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Contraction elements per stage: the TMA coordinate counts elements,
  // 128 for int8, 64 for bf16 (128 bytes either way).
  static_assert(!F16 || (!A_MN && !B_MN), "bf16 operands are read K-major");
  constexpr int KE = F16 ? BK / 2 : BK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the previous kernel's outputs (operands) are visible from here
  const uint32_t tmem_base = *tmem_slot;
  // Contraction splits of kps k-blocks each (one split unless the
  // contraction exceeds the int32-safe length); tile t is split t / per_split.
  const int per_split = tiles_per_split(tiles_m, tiles_n, group);
  const int num_tiles = per_split * ((kblocks + kps - 1) / kps);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int tm, tn;
        const int sp = t / per_split;
        tile_coords(t - sp * per_split, tiles_m, tiles_n, group, tm, tn);
        const int kb1 = min(kblocks, (sp + 1) * kps);
        for (int kb = sp * kps; kb < kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          // A K-major output slab of fewer than 128 rows is loaded as a box of
          // a_box_rows rows; the accumulator rows past it are never stored.
          mbar_arrive_expect_tx(fb, STAGE_BYTES - (BM - a_box_rows) * BK);
          const uint32_t a_dst = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_BYTES);
          if (A_MN) tma_load_2d(a_dst, &tmA, fb, tm * BM, kb * BK);
          else tma_load_2d(a_dst, &tmA, fb, kb * KE, tm * BM);
          if (B_MN) {
            tma_load_2d(b_dst, &tmB, fb, tn * BN, kb * BK);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB, fb, tn * BN + 128, kb * BK);
          } else {
            tma_load_2d(b_dst, &tmB, fb, kb * KE, tn * BN);
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every copy issued must have landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (issued & (1u << s)) mbar_wait_drain(full0 + 8 * s, (issued_phase >> s) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = F16 ? idesc_bf16(BM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0)
                                     : idesc_i8(BM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int kb0 = (t / per_split) * kps;
        const int kb1 = min(kblocks, kb0 + kps);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // K-major: advance 32 bytes inside the 128-byte swizzle row.
            // MN-major: advance 32 contraction rows of 128 bytes.
            const uint64_t a_desc = A_MN ? smem_desc_sw128(a_base + kk * 4096, 16384, 1024)
                                         : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t b_desc = B_MN ? smem_desc_sw128(b_base + kk * 4096, 16384, 1024)
                                         : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            if constexpr (F16) mma_bf16(d_tmem, a_desc, b_desc, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
            else mma_i8(d_tmem, a_desc, b_desc, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          mma_commit(empty0 + 8 * stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(tfull0 + 8 * acc);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      // All issued MMAs must be complete before TMEM is released.
      mma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int tm, tn;
      const int sp = t / per_split;
      tile_coords(t - sp * per_split, tiles_m, tiles_n, group, tm, tn);
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      Epi eps = ep;
      eps.out = reinterpret_cast<OutT*>(ep.out) + sp * ep.split_stride;
      if constexpr (std::is_same<OutT, int32_t>::value)
        epilogue_tile_raw<BN>(eps, tmem_base + acc * BN, quarter, lane, tm * BM, tn * BN);
      else
        epilogue_tile<OutT, HB, F16, BN>(eps, tmem_base + acc * BN, quarter, lane, tm * BM, tn * BN,
                                         epi_stage + quarter * kEpiStageFloats);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ CTA pairs
// The same GEMM on 256x256 tiles computed by a cluster of two CTAs on two
// SMs (tcgen05 cta_group::2).  Each CTA loads 128 rows of A and 128 of the
// 256 B columns per stage (32 KB; TMA loads without multicast, counted on the
// even CTA's barrier), so per SM the operand traffic through shared memory
// is 64 B/clk at full MMA rate instead of 96 for a 128x256 tile on one SM;
// the even CTA issues the 256x256x32 MMAs and commits to both CTAs'
// barriers; each CTA drains its own 128 accumulator rows.
constexpr int PSTAGES = 6;
constexpr int PA_BYTES = 128 * BK;                 // 16 KiB: this CTA's A rows
constexpr int PB_BYTES = 128 * BK;                 // 16 KiB: this CTA's B columns
constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;  // 32 KiB
constexpr int PNUM_BARS = 2 * PSTAGES + 5;
constexpr int PSMEM_BYTES = 1024 + PSTAGES * PSTAGE_BYTES + 8 * PNUM_BARS + 16 + kEpiStageBytes;

template <bool A_MN, bool B_MN, typename OutT, int HB, bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, int tiles_m, int tiles_n,
                        int kblocks, int kps, int group, Epi ep, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + PSTAGES * PA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + PSTAGES * PB_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + PNUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(tmem_slot + 4);  // scalar accesses only

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + PSTAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * PSTAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * PSTAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * PSTAGES + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  static_assert(!F16 || (!A_MN && !B_MN), "bf16 operands are read K-major");
  constexpr int KE = F16 ? BK / 2 : BK;  // contraction elements per stage
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);   // rank 0's: its expect_tx arrival + both CTAs' bytes
      mbar_init(empty0 + 8 * s, 1);  // the pair's MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);   // the pair's MMA commit
      mbar_init(tempty0 + 8 * a, 8);  // rank 0's: 4 epilogue warps of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  griddep_wait();  // the previous kernel's outputs (operands) are visible from here
  const uint32_t tmem_base = *tmem_slot;
  // Contraction splits of kps k-blocks each (one split unless the
  // contraction exceeds the int32-safe length); tile t is split t / per_split.
  const int per_split = tiles_per_split(tiles_m, tiles_n, group);
  const int num_tiles = per_split * ((kblocks + kps - 1) / kps);
  const uint32_t lead_full0 = mapa_shared(full0, 0);
  const uint32_t lead_tempty0 = mapa_shared(tempty0, 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, armed = 0, armed_phase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += npairs) {
        int tm, tn;
        const int sp = t / per_split;
        tile_coords(t - sp * per_split, tiles_m, tiles_n, group, tm, tn);
        const int a_row = tm * 256 + static_cast<int>(rank) * 128;
        const int b_col = tn * 256 + static_cast<int>(rank) * 128;
        const int kb0 = sp * kps, kb1 = min(kblocks, (sp + 1) * kps);
        // Integer products: every other tile of this pair walks its
        // contraction backwards, so it starts on the k-slices the tiles just
        // finished (same operand rows for the next tiles of a group) while
        // they are still in L2; int32 sums are exact in any order.  The MMA
        // issuer takes the stages as they come (its first stage initialises).
        const bool back = !F16 && (((t - pair) / npairs) & 1);
        for (int i = 0; i < kb1 - kb0; ++i) {
          const int kb = back ? kb1 - 1 - i : kb0 + i;
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) {
            mbar_arrive_expect_tx(full0 + 8 * stage, 2 * PSTAGE_BYTES);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fb = lead_full0 + 8 * stage;
          const uint32_t a_dst = smem_u32(sA + stage * PA_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * PB_BYTES);
          if (A_MN) tma_load_2d_pair(a_dst, &tmA, fb, a_row, kb * BK);
          else tma_load_2d_pair(a_dst, &tmA, fb, kb * KE, a_row);
          if (B_MN) tma_load_2d_pair(b_dst, &tmB, fb, b_col, kb * BK);
          else tma_load_2d_pair(b_dst, &tmB, fb, kb * KE, b_col);
          if (++stage == PSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (rank == 0) {
        // Every stage armed here counts both CTAs' copies: wait for them.
        for (int s = 0; s < PSTAGES; ++s)
          if (armed & (1u << s)) mbar_wait_drain(full0 + 8 * s, (armed_phase >> s) & 1u);
      } else if (!ok) {
        __nanosleep(100000);  // give copies in flight time to land before exit
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = F16 ? idesc_bf16(256, 256, A_MN ? 1 : 0, B_MN ? 1 : 0)
                                     : idesc_i8(256, 256, A_MN ? 1 : 0, B_MN ? 1 : 0);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += npairs) {
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int kb0 = (t / per_split) * kps;
        const int kb1 = min(kblocks, kb0 + kps);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * PA_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * PB_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t a_desc = A_MN ? smem_desc_sw128(a_base + kk * 4096, 16384, 1024)
                                         : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t b_desc = B_MN ? smem_desc_sw128(b_base + kk * 4096, 16384, 1024)
                                         : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            if constexpr (F16) mma_bf16_pair(d_tmem, a_desc, b_desc, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
            else mma_i8_pair(d_tmem, a_desc, b_desc, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          mma_commit_pair_mc(empty0 + 8 * stage, 0x3);
          if (++stage == PSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(tfull0 + 8 * acc, 0x3);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      mma_commit_pair_mc(drain, 0x1);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    uint32_t acc = 0, acc_phase = 0;
    for (int t = pair; t < num_tiles; t += npairs) {
      int tm, tn;
      const int sp = t / per_split;
      tile_coords(t - sp * per_split, tiles_m, tiles_n, group, tm, tn);
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      Epi eps = ep;
      eps.out = reinterpret_cast<OutT*>(ep.out) + sp * ep.split_stride;
      if constexpr (std::is_same<OutT, int32_t>::value)
        epilogue_tile_raw(eps, tmem_base + acc * BN, quarter, lane,
                          tm * 256 + static_cast<int>(rank) * 128, tn * BN);
      else
        epilogue_tile<OutT, HB, F16>(eps, tmem_base + acc * BN, quarter, lane,
                                     tm * 256 + static_cast<int>(rank) * 128, tn * BN,
                                     epi_stage + quarter * kEpiStageFloats);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_tempty0 + 8 * acc);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  griddep_launch_dependents();
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the pair may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(status, 1 << QL_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ a few rows
// The forward at up to 4 tokens is a stream of the whole weight with at most
// 4 multiply-adds per weight byte: a 128-row tensor-core tile would spend
// its time on rows that do not exist.  One warp per weight row n: each lane
// streams 16-byte pieces of the row (evict-first), multiplies them with the
// same pieces of every token's codes (__dp4a: 4 int8 products into an int32
// sum, exact), the warp adds its lanes' sums (redux.sync, exact), and lane m
// writes y[m, n] = ((float)acc * row_scale[m]) * col_scale[n] + bias[n], the
// epilogue of the tile kernel.
template <int MT, typename OutT>
__global__ void __launch_bounds__(256) gemv_i8_kernel(
    const int8_t* __restrict__ xq, int64_t ldx, int M, const int8_t* __restrict__ wq,
    int64_t ldw, int N, int K, const float* __restrict__ row_scale,
    const float* __restrict__ col_scale, const float* __restrict__ bias, OutT* __restrict__ out,
    int64_t ldo) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); n < N; n += nwarps) {
    const int8_t* wrow = wq + n * ldw;
    int acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
#pragma unroll 4
    for (int k0 = lane * 16; k0 < K; k0 += 512) {
      const int4 w = __ldcs(reinterpret_cast<const int4*>(wrow + k0));
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const int4 x = __ldg(reinterpret_cast<const int4*>(xq + m * ldx + k0));
          acc[m] = __dp4a(w.x, x.x, acc[m]);
          acc[m] = __dp4a(w.y, x.y, acc[m]);
          acc[m] = __dp4a(w.z, x.z, acc[m]);
          acc[m] = __dp4a(w.w, x.w, acc[m]);
        }
      }
    }
    int mine = 0;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int t = __reduce_add_sync(0xFFFFFFFFu, acc[m]);
      if (lane == m) mine = t;
    }
    if (lane < M) {
      float v = __int2float_rn(mine) * (row_scale ? row_scale[lane] : 1.0f);
      if (col_scale) v = v * col_scale[n];
      if (bias) v = v + bias[n];
      if constexpr (sizeof(OutT) == 4) out[lane * ldo + n] = v;
      else out[lane * ldo + n] = __float2bfloat16_rn(v);
    }
  }
}

template <int MT>
cudaError_t run_gemv(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb, int64_t rows,
                     int64_t cols, int64_t kc, const GemmEpilogue& e, cudaStream_t s) {
  const int grid = static_cast<int>(std::min<int64_t>((cols + 7) / 8, device_info().sms * 8));
  cudaEvent_t before = nullptr, after = nullptr;
  gemm_timing_events(&before, &after);
  if (before) cudaEventRecord(before, s);
  if (e.out_bf16)
    gemv_i8_kernel<MT, __nv_bfloat16><<<grid, 256, 0, s>>>(
        A, lda, static_cast<int>(rows), B, ldb, static_cast<int>(cols), static_cast<int>(kc),
        e.row_scale, e.col_scale, e.bias, reinterpret_cast<__nv_bfloat16*>(e.out), e.ldo);
  else
    gemv_i8_kernel<MT, float><<<grid, 256, 0, s>>>(
        A, lda, static_cast<int>(rows), B, ldb, static_cast<int>(cols), static_cast<int>(kc),
        e.row_scale, e.col_scale, e.bias, reinterpret_cast<float*>(e.out), e.ldo);
  cudaError_t err = cudaGetLastError();
  if (after) cudaEventRecord(after, s);
  count_launches(1);
  return err;
}

// ------------------------------------------------------------------ host
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Rows of the K-major A box: a slab of fewer than 128 output rows loads only
// its rows (rounded up to 16) instead of a mostly zero-filled 128-row box.
int a_box_rows(int64_t rows) {
  return rows >= BM ? BM : static_cast<int>(std::max<int64_t>(16, (rows + 15) / 16 * 16));
}

// 2-D int8 tensor [outer][inner] with the given row pitch; boxes of
// box_inner x box_outer bytes, 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
               uint32_t box_inner, uint32_t box_outer) {
  return encode_tmap_2d(m, 1, base, inner, outer, pitch, box_inner, box_outer, true);
}

// Clusters of two that can be resident together (cached per device).
template <typename K>
int pair_slots(K kern) {
  static int slots[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64) {
    const int cached = __atomic_load_n(&slots[dev], __ATOMIC_ACQUIRE);
    if (cached > 0) return cached;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PSMEM_BYTES;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1)
    n = device_info().sms / 2;
  if (dev < 64) __atomic_store_n(&slots[dev], n, __ATOMIC_RELEASE);
  return n;
}

template <bool A_MN, bool B_MN, typename OutT, int HB, bool F16 = false>
cudaError_t run_pair(const CUtensorMap& ta, const CUtensorMap& tb, int tiles_m, int tiles_n,
                     int kblocks, int kps, const Epi& ep, int32_t* status, cudaStream_t s,
                     bool upper = false) {
  auto kern = gemm_i8_pair_kernel<A_MN, B_MN, OutT, HB, F16>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !__atomic_load_n(&configured[dev], __ATOMIC_ACQUIRE)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PSMEM_BYTES);
    if (e != cudaSuccess) return e;
    __atomic_store_n(&configured[dev], 1, __ATOMIC_RELEASE);
  }
  const int per_split = upper ? tiles_m * (tiles_m + 1) / 2 : tiles_m * tiles_n;
  const int tiles = per_split * ((kblocks + kps - 1) / kps);
  const int slots = pair_slots(kern);
  const int pairs = tiles < slots ? tiles : slots;
  cudaEvent_t before = nullptr, after = nullptr;
  gemm_timing_events(&before, &after);
  if (before) cudaEventRecord(before, s);
  cudaError_t e = launch_pdl(kern, dim3(2 * pairs), dim3(NUM_THREADS), PSMEM_BYTES, s, ta, tb,
                             tiles_m, tiles_n, kblocks, kps, upper ? 0 : (A_MN ? 16 : 1), ep,
                             status);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (after) cudaEventRecord(after, s);
  count_launches(1);
  return e;
}

template <bool A_MN, bool B_MN, typename OutT, int HB, bool F16 = false, int TBN = 256>
cudaError_t run(const CUtensorMap& ta, const CUtensorMap& tb, int tiles_m, int tiles_n,
                int kblocks, int kps, const Epi& ep, int32_t* status, cudaStream_t s) {
  auto kern = gemm_i8_kernel<A_MN, B_MN, OutT, HB, F16, TBN>;
  constexpr int SMEM_BYTES = Single<TBN>::kSmemBytes;
  // Opt in to the large dynamic shared memory once per device.
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !__atomic_load_n(&configured[dev], __ATOMIC_ACQUIRE)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    __atomic_store_n(&configured[dev], 1, __ATOMIC_RELEASE);
  }
  const int tiles = tiles_m * tiles_n * ((kblocks + kps - 1) / kps);
  const int sms = device_info().sms;
  const int grid = tiles < sms ? tiles : sms;
  cudaEvent_t before = nullptr, after = nullptr;
  gemm_timing_events(&before, &after);
  if (before) cudaEventRecord(before, s);
  cudaError_t e = launch_pdl(kern, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, s, ta, tb, tiles_m,
                             tiles_n, kblocks, kps, A_MN ? 16 : 1,
                             A_MN ? BM : a_box_rows(ep.rows), ep, status);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (after) cudaEventRecord(after, s);
  count_launches(1);
  return e;
}

template <bool A_MN, bool B_MN, typename OutT, int HB, bool F16 = false>
cudaError_t go(bool pair, const CUtensorMap& ta, const CUtensorMap& tb, int tiles_m, int tiles_n,
               int kblocks, const Epi& ep, int32_t* status, cudaStream_t s, int kps = 0,
               bool upper = false) {
  if (kps <= 0) kps = kblocks;
  if (pair)
    return run_pair<A_MN, B_MN, OutT, HB, F16>(ta, tb, tiles_m, tiles_n, kblocks, kps, ep, status,
                                               s, upper);
  return run<A_MN, B_MN, OutT, HB, F16>(ta, tb, tiles_m, tiles_n, kblocks, kps, ep, status, s);
}

cudaError_t dispatch_dx(bool pair, const CUtensorMap& ta, const CUtensorMap& tb, int tiles_m,
                        int tiles_n, int kblocks, const Epi& ep, bool bf16, int hb,
                        int32_t* status, cudaStream_t s) {
#define QL_RUN(T, H) return go<false, true, T, H>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s)
  if (bf16) {
    switch (hb) {
      case 0: QL_RUN(__nv_bfloat16, 0);
      case 2: QL_RUN(__nv_bfloat16, 2);
      case 4: QL_RUN(__nv_bfloat16, 4);
      case 8: QL_RUN(__nv_bfloat16, 8);
      case 16: QL_RUN(__nv_bfloat16, 16);
      case 32: QL_RUN(__nv_bfloat16, 32);
      case 64: QL_RUN(__nv_bfloat16, 64);
      case 128: QL_RUN(__nv_bfloat16, 128);
    }
  } else {
    switch (hb) {
      case 0: QL_RUN(float, 0);
      case 2: QL_RUN(float, 2);
      case 4: QL_RUN(float, 4);
      case 8: QL_RUN(float, 8);
      case 16: QL_RUN(float, 16);
      case 32: QL_RUN(float, 32);
      case 64: QL_RUN(float, 64);
      case 128: QL_RUN(float, 128);
    }
  }
#undef QL_RUN
  return cudaErrorInvalidValue;
}

}  // namespace

bool encode_tmap_2d(CUtensorMap* m, int elem_bytes, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                    bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap(CUtensorMap* m, int elem_bytes, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, b, e,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_rows_128b(CUtensorMap* m, int elem_bytes, const void* base, uint64_t cols,
                      uint64_t rows, uint64_t pitch, uint32_t box_rows) {
  // [rows][cols / L][L] with L elements = 128 bytes per line; one box is
  // box_rows whole rows, written to shared memory with the 128-byte swizzle.
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t L = 128 / static_cast<uint64_t>(elem_bytes);
  if (cols % L != 0 || cols / L > 256) return false;
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const cuuint64_t dims[3] = {L, cols / L, rows};
  const cuuint64_t strides[2] = {128, pitch};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(L), static_cast<cuuint32_t>(cols / L), box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_i8(const int8_t* A, bool a_mn, int64_t lda, const int8_t* B, bool b_mn,
                           int64_t ldb, int64_t rows, int64_t cols, int64_t kc,
                           const GemmEpilogue& e, int32_t* status, cudaStream_t s) {
  // Up to 4 rows of K-major x K-major (the forward at a few tokens): one
  // warp per output column on the CUDA cores, a single pass over B.  (Every
  // row re-reads its piece of A per B row, so past a few rows the tensor-core
  // tile is faster again.)
  if (!a_mn && !b_mn && e.hb == 0 && rows <= 4 && kc % 16 == 0 && lda % 16 == 0 && ldb % 16 == 0) {
    if (rows <= 1) return run_gemv<1>(A, lda, B, ldb, rows, cols, kc, e, s);
    if (rows <= 2) return run_gemv<2>(A, lda, B, ldb, rows, cols, kc, e, s);
    return run_gemv<4>(A, lda, B, ldb, rows, cols, kc, e, s);
  }
  // Outputs with more than one 128-row slab run on CTA pairs (256x256
  // tiles); smaller ones on single CTAs (128x256 tiles, or 128x64 when the
  // wide tiles would occupy fewer than half the SMs: the forward at a few
  // tokens is a stream of the whole weight and wants every SM on it).
  const bool pair = rows > BM;
  const bool narrow = !pair && !a_mn && !b_mn && e.hb == 0 &&
                      2 * ((cols + BN - 1) / BN) < device_info().sms;
  CUtensorMap ta, tb;
  const bool ok_a = a_mn ? make_tmap(&ta, A, rows, kc, lda, 128, BK)
                         : make_tmap(&ta, A, kc, rows, lda, BK, pair ? BM : a_box_rows(rows));
  const bool ok_b = b_mn ? make_tmap(&tb, B, cols, kc, ldb, 128, BK)
                         : make_tmap(&tb, B, kc, cols, ldb, BK, pair ? 128 : narrow ? 64 : BN);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  Epi ep{};
  ep.out = e.out;
  ep.ldo = e.ldo;
  ep.split_stride = 0;
  ep.rows = static_cast<int>(rows);
  ep.cols = static_cast<int>(cols);
  ep.row_scale = e.row_scale;
  ep.col_scale = e.col_scale;
  ep.bias = e.bias;
  ep.hc = e.hc;
  const int tile_rows = pair ? 2 * BM : BM;
  const int tiles_m = static_cast<int>((rows + tile_rows - 1) / tile_rows);
  const int tiles_n = static_cast<int>((cols + BN - 1) / BN);
  const int kblocks = static_cast<int>((kc + BK - 1) / BK);
  const bool bf16 = e.out_bf16 != 0;
  // The layer's three products: forward (K-major x K-major), input gradient
  // (K-major x MN-major, optional fused rotation), weight gradient
  // (MN-major x MN-major, float32 out).
  if (narrow) {
    const int tn64 = static_cast<int>((cols + 63) / 64);
    if (bf16) return run<false, false, __nv_bfloat16, 0, false, 64>(ta, tb, tiles_m, tn64, kblocks, kblocks, ep, status, s);
    return run<false, false, float, 0, false, 64>(ta, tb, tiles_m, tn64, kblocks, kblocks, ep, status, s);
  }
  if (!a_mn && !b_mn && e.hb == 0) {
    if (bf16) return go<false, false, __nv_bfloat16, 0>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s);
    return go<false, false, float, 0>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s);
  }
  if (!a_mn && b_mn) return dispatch_dx(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, bf16, e.hb, status, s);
  if (a_mn && b_mn && e.hb == 0 && !bf16)
    return go<true, true, float, 0>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_bf16(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t rows,
                             int64_t cols, int64_t kc, const GemmEpilogue& e, int32_t* status,
                             cudaStream_t s, bool* upper_only) {
  // Both operands K-major bf16: a 128-byte stage row holds 64 elements and
  // each kind::f16 MMA consumes K = 16 (32 bytes), the same byte layout as
  // the int8 path.
  const bool pair = rows > BM;
  const bool narrow = !pair && 2 * ((cols + BN - 1) / BN) < device_info().sms;
  CUtensorMap ta, tb;
  const bool ok_a = encode_tmap_2d(&ta, 2, A, static_cast<uint64_t>(kc), static_cast<uint64_t>(rows),
                                   static_cast<uint64_t>(lda) * 2, BK / 2,
                                   pair ? BM : a_box_rows(rows), true);
  const bool ok_b = encode_tmap_2d(&tb, 2, B, static_cast<uint64_t>(kc), static_cast<uint64_t>(cols),
                                   static_cast<uint64_t>(ldb) * 2, BK / 2,
                                   pair ? 128 : narrow ? 64 : BN, true);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  Epi ep{};
  ep.out = e.out;
  ep.ldo = e.ldo;
  ep.split_stride = 0;
  ep.rows = static_cast<int>(rows);
  ep.cols = static_cast<int>(cols);
  ep.row_scale = e.row_scale;
  ep.col_scale = e.col_scale;
  ep.bias = e.bias;
  ep.hc = e.hc;
  const int tile_rows = pair ? 2 * BM : BM;
  const int tiles_m = static_cast<int>((rows + tile_rows - 1) / tile_rows);
  const int tiles_n = static_cast<int>((cols + BN - 1) / BN);
  const int kblocks = static_cast<int>((kc + BK / 2 - 1) / (BK / 2));
  if (e.hb != 0) return cudaErrorInvalidValue;
  if (e.ns_x || e.ns_xt || e.ns_mirror) {
    // The Newton-Schulz epilogue: bf16 output, 16-byte pieces of ns_x, out
    // and ns_xt rows (pitches multiples of 8 elements, rows a multiple of 16);
    // a transposed copy into ns_xt needs ns_x, ns_mirror a symmetric product.
    if (!e.out_bf16 || e.row_scale || e.col_scale || e.bias || (e.ldo % 8) != 0 ||
        (rows % 16) != 0 || (cols % 16) != 0 || (reinterpret_cast<uintptr_t>(e.out) & 15) ||
        (e.ns_x && (reinterpret_cast<uintptr_t>(e.ns_x) & 15)) ||
        (e.ns_xt && (!e.ns_x || e.ns_mirror || (e.ns_ldt % 8) != 0 ||
                     (reinterpret_cast<uintptr_t>(e.ns_xt) & 15))) ||
        (e.ns_mirror && !(upper_only && *upper_only)))
      return cudaErrorInvalidValue;
    ep.ns_x = reinterpret_cast<const __nv_bfloat16*>(e.ns_x);
    ep.ns_xt = reinterpret_cast<__nv_bfloat16*>(e.ns_xt);
    ep.ns_ldt = e.ns_ldt;
    ep.ns_a = e.ns_a;
    ep.ns_c = e.ns_c;
  }
  if (narrow) {
    if (upper_only) *upper_only = false;  // every tile is computed
    const int tn64 = static_cast<int>((cols + 63) / 64);
    if (e.out_bf16)
      return run<false, false, __nv_bfloat16, 0, true, 64>(ta, tb, tiles_m, tn64, kblocks, kblocks, ep, status, s);
    return run<false, false, float, 0, true, 64>(ta, tb, tiles_m, tn64, kblocks, kblocks, ep, status, s);
  }
  // A symmetric product (the caller passes upper_only set): with CTA-pair
  // tiles on a square grid only the upper tiles are computed, and
  // *upper_only stays true to tell the caller to fill the lower ones.
  const bool upper = upper_only && *upper_only && pair && rows == cols;
  if (upper_only) *upper_only = upper;
  // The lower tiles are mirrored only when the product runs on its upper
  // tiles (otherwise every tile is computed).
  ep.ns_mirror = e.ns_mirror && upper ? 1 : 0;
  if (e.out_bf16)
    return go<false, false, __nv_bfloat16, 0, true>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep,
                                                   status, s, 0, upper);
  return go<false, false, float, 0, true>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s,
                                          0, upper);
}

// ------------------------------------------------------------------ long contractions
// Sum of the int32 partial products of every split in int64, then the
// epilogue of launch_gemm_i8: ((float)acc * row_scale) * col_scale + bias.
// One thread per 4 consecutive outputs.
template <typename OutT>
__global__ void __launch_bounds__(256) combine_splits_kernel(
    const int32_t* __restrict__ parts, int splits, int64_t split_stride, int64_t rows, int cols,
    const float* __restrict__ row_scale, const float* __restrict__ col_scale,
    const float* __restrict__ bias, OutT* __restrict__ out, int64_t ldo) {
  const int64_t quads = rows * (cols / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < quads;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / (cols / 4);
    const int c = static_cast<int>(i - r * (cols / 4)) * 4;
    long long acc[4] = {0, 0, 0, 0};
    for (int sp = 0; sp < splits; ++sp) {
      const int4 p = __ldcs(reinterpret_cast<const int4*>(parts + sp * split_stride + r * cols + c));
      acc[0] += p.x;
      acc[1] += p.y;
      acc[2] += p.z;
      acc[3] += p.w;
    }
    const float rs = row_scale ? row_scale[r] : 1.0f;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = __ll2float_rn(acc[e]) * rs;
      if (col_scale) v[e] = v[e] * col_scale[c + e];
      if (bias) v[e] = v[e] + bias[c + e];
    }
    OutT* o = out + r * ldo + c;
    if constexpr (sizeof(OutT) == 4) {
      *reinterpret_cast<float4*>(o) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
      *reinterpret_cast<uint2*>(o) = make_uint2(bf16x2(v[0], v[1]), bf16x2(v[2], v[3]));
    }
  }
}

int small_output_splits(int64_t rows, int64_t cols, int64_t kc) {
  // Splits that bring a one-slab output (rows <= 128) to about one wave.
  if (rows > BM) return 1;
  const int64_t tiles = (cols + BN - 1) / BN;
  const int64_t kblocks = (kc + BK - 1) / BK;
  int64_t sp = device_info().sms / tiles;
  sp = std::min<int64_t>(std::min<int64_t>(sp, kMaxSmallSplits), kblocks / 4);
  return static_cast<int>(std::max<int64_t>(sp, 1));
}

int contraction_splits(int64_t kc) {
  const int64_t kblocks = (kc + BK - 1) / BK;
  return static_cast<int>((kblocks + kMaxSplitBlocks - 1) / kMaxSplitBlocks);
}

cudaError_t launch_gemm_i8_long(const int8_t* A, bool a_mn, int64_t lda, const int8_t* B, bool b_mn,
                                int64_t ldb, int64_t rows, int64_t cols, int64_t kc,
                                int32_t* parts, size_t parts_elems, const GemmEpilogue& e,
                                int32_t* status, cudaStream_t s, int min_splits) {
  // The contraction in splits of at most kMaxSplitBlocks * 128 = 130,944
  // elements (at least min_splits of them, to spread a small output over
  // more SMs), each written as raw int32 partial sums [split][rows][cols];
  // then one pass sums the splits in int64 and applies the epilogue.
  if (e.hb != 0 || cols % 16 != 0) return cudaErrorInvalidValue;
  const bool pair = rows > BM;
  CUtensorMap ta, tb;
  const bool ok_a = a_mn ? make_tmap(&ta, A, rows, kc, lda, 128, BK)
                         : make_tmap(&ta, A, kc, rows, lda, BK, pair ? BM : a_box_rows(rows));
  const bool ok_b = b_mn ? make_tmap(&tb, B, cols, kc, ldb, 128, BK)
                         : make_tmap(&tb, B, kc, cols, ldb, BK, pair ? 128 : BN);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  Epi ep{};
  ep.out = parts;
  ep.ldo = cols;
  ep.split_stride = rows * cols;
  ep.rows = static_cast<int>(rows);
  ep.cols = static_cast<int>(cols);
  const int tile_rows = pair ? 2 * BM : BM;
  const int tiles_m = static_cast<int>((rows + tile_rows - 1) / tile_rows);
  const int tiles_n = static_cast<int>((cols + BN - 1) / BN);
  const int kblocks = static_cast<int>((kc + BK - 1) / BK);
  const int splits = std::max(contraction_splits(kc), std::min(min_splits, kblocks));
  const int kps = (kblocks + splits - 1) / splits;
  const int nsp = (kblocks + kps - 1) / kps;  // splits actually written
  if (static_cast<size_t>(nsp) * static_cast<size_t>(rows) * static_cast<size_t>(cols) > parts_elems)
    return cudaErrorInvalidValue;  // the partial sums would not fit
  cudaError_t err;
  if (!a_mn && b_mn)
    err = go<false, true, int32_t, 0>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s, kps);
  else if (a_mn && b_mn)
    err = go<true, true, int32_t, 0>(pair, ta, tb, tiles_m, tiles_n, kblocks, ep, status, s, kps);
  else
    return cudaErrorInvalidValue;
  if (err != cudaSuccess) return err;
  const int64_t quads = rows * (cols / 4);
  const int grid = static_cast<int>(std::min<int64_t>((quads + 255) / 256, device_info().sms * 8));
  if (e.out_bf16)
    combine_splits_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        parts, nsp, rows * cols, rows, static_cast<int>(cols), e.row_scale, e.col_scale, e.bias,
        reinterpret_cast<__nv_bfloat16*>(e.out), e.ldo);
  else
    combine_splits_kernel<float><<<grid, 256, 0, s>>>(
        parts, nsp, rows * cols, rows, static_cast<int>(cols), e.row_scale, e.col_scale, e.bias,
        reinterpret_cast<float*>(e.out), e.ldo);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ql
