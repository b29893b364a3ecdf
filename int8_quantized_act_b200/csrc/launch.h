// launch.h - host-side launchers of the CUDA kernels, called by the C ABI
// (qlinear_api.cu) after it has validated every argument.  Each returns the
// launch's cudaError_t; none allocates, none synchronizes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace ql {

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;  // max dynamic shared memory per block (opt-in), bytes
};
const DeviceInfo& device_info();  // current device, cached

// Launch accounting (ql_kernel_launches) and the GEMM timing events
// (ql_set_gemm_timing_events) of the calling thread.
void count_launches(int n);

// Launch kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization: it may start while the previous kernel on the stream
// finishes (its prologue overlaps that kernel's tail) and calls
// griddep_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
void gemm_timing_events(cudaEvent_t* before, cudaEvent_t* after);

// 2-D tensor map over a row-major [outer][inner] array of elem_bytes-byte
// elements (raw bits; the pitch in bytes), boxes of box_inner x box_outer
// elements, out-of-range elements read as zero; 128-byte swizzle or none.
// Whole rows as [rows][cols / L][L] (L elements = one 128-byte line; cols a
// multiple of L, at most 256 lines), boxes of box_rows rows, 128-byte swizzle.
// Any rank (1..5): dims[0] innermost (elements), strides[i] the byte pitch of
// dimension i + 1 (rank - 1 of them), box the copied extent per dimension.
bool encode_tmap(CUtensorMap* m, int elem_bytes, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128);
bool encode_rows_128b(CUtensorMap* m, int elem_bytes, const void* base, uint64_t cols,
                      uint64_t rows, uint64_t pitch, uint32_t box_rows);
bool encode_tmap_2d(CUtensorMap* m, int elem_bytes, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                    bool swizzle128);

// The host checks of qlinear_bwd_dx that come before its workspace is looked
// at, in its order (argument, shape, then null pointers): returns the status
// code, and sets *noop when the call has nothing to compute (M == 0 or K == 0).
int check_bwd_dx_args(const void* dy, int dyt, int64_t M, int64_t N, const int8_t* wq,
                      const float* sw, int64_t K, int hadamard_block, const void* dx, int dxt,
                      const int32_t* d_status, bool* noop);

// -------------------------------------------------------------- row kernels
// Per-row quantization (optionally scaled per column and rotated); see
// qlinear_quantize_rows.  xt: 0 = float32, 1 = bf16.
cudaError_t launch_quant_rows(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                              const float* col_scale, int B, float hc, unsigned flags,
                              int8_t* q, int64_t ldq, float* row_scale, int32_t* status,
                              cudaStream_t s);

// The same quantization for bf16 rows of 128..16384 columns (a multiple of
// 128) and blocks B <= 128 without a column scale, two threads per
// 128-column block, rows in and codes out by TMA: eligible when there are
// enough rows to give every SM a tile.  Launched by launch_quant_rows.
bool quant_blk_eligible(int64_t rows, int64_t cols, int64_t ldx, int B, bool col_scale);
cudaError_t launch_quant_blk(const void* x, int64_t rows, int64_t cols, int64_t ldx, int B,
                             float hc, unsigned flags, int8_t* q, int64_t ldq, float* rs,
                             int32_t* st, cudaStream_t s);

// y = x R per row (x may equal y).  xt / yt: 0 = float32, 1 = bf16.
cudaError_t launch_hadamard(const void* x, int xt, int64_t ldx, void* y, int yt, int64_t ldy,
                            int64_t rows, int64_t cols, int B, float hc, cudaStream_t s);

// w[r,:] = s[r] * q[r,:] in float32, then times R for B > 0 (hc = fl32(1/sqrt(B))).
cudaError_t launch_dequant_rows(const int8_t* q, int64_t ldq, const float* s, void* w, int wt,
                                int64_t ldw, int64_t rows, int64_t cols, int B, float hc,
                                cudaStream_t st);

// Column statistics of t = dY[m,n]*s_x[m]: colmax[n] = bits of max|t|
// (atomicMax; caller zeroes), colsum[n] += sum_m dY[m,n] in float64.  With
// rowmax != NULL also rowmax[m] = bits of max_n |dY[m,n]*sw[n]| (caller zeroes).
cudaError_t launch_colstats(const void* dy, int dyt, int64_t M, int64_t N, const float* sx,
                            uint32_t* colmax, double* colsum, const float* sw, uint32_t* rowmax,
                            int32_t* status, cudaStream_t s);

// Zero colmax [N], colsum [N] and (if rowmax != NULL) rowmax [M] in one launch.
cudaError_t launch_zero_stats(uint32_t* colmax, double* colsum, int64_t N, uint32_t* rowmax,
                              int64_t M, cudaStream_t s);

// From the statistics pass's maxima (float bits; a zero maximum gives zero
// factors and scales): q2 = rne((dY*rs2[m]) * (127/colmax[n])) and, if
// q1 != NULL, q1 = rne((dY*cs1[n]) * (127/rowmax[m])), both [M,N] (dY streamed
// through shared memory by TMA); also s2 = colmax/127, db = colsum (if db)
// and, with q1, s1 = rowmax/127.
cudaError_t launch_dualquant(const void* dy, int dyt, int64_t M, int64_t N, const float* cs1,
                             const float* rs2, const uint32_t* colmax, const double* colsum,
                             const uint32_t* rowmax, float* s1, float* s2, float* db, int8_t* q1,
                             int8_t* q2, int32_t* status, cudaStream_t s);

// out[r, :] = bias (or 0), dtype ot; used when the contraction is empty.
cudaError_t launch_fill_rows(void* out, int ot, int64_t rows, int64_t cols, const float* bias,
                             cudaStream_t s);

// -------------------------------------------------------------- MuonAuxAdamW
// Workspace of the Newton-Schulz iteration for an [N, K] weight (r = min,
// c = max of N, K): ||U||^2, X [r, c] bf16 and two buffers of X^T [c, r] bf16
// (each step reads one and writes the other), A and B [r, r] bf16; byte
// offsets, each 256-byte aligned.
struct MuonLayout {
  int64_t sumsq, X, Xt, Xt2, A, Bm, total;
};
MuonLayout muon_layout(int64_t N, int64_t K);
// M <- beta*M + (1-beta)*G; O [N, K] bf16 <- NS(U) after `steps` (>= 1) steps.
cudaError_t launch_muon_orthogonalize(const float* grad, float* mom, int64_t N, int64_t K,
                                      float beta, int steps, void* O, void* ws, int32_t* status,
                                      cudaStream_t s);
// p <- AdamW(p, g) elementwise (m, v in place), the constants of UpdateConsts.
struct UpdateConsts;
cudaError_t launch_adamw_vector(float* p, const float* g, float* m, float* v, int64_t n,
                                const UpdateConsts& c, int32_t* status, cudaStream_t s);
// w = s*q; w' = w*a - st*O (O bf16 [N, K]); per-row stochastic requantization.
cudaError_t launch_update_dir(int8_t* wq, float* sw, const void* O, int64_t N, int64_t K, float a,
                              float st, uint64_t seed, uint64_t step, int32_t* status,
                              cudaStream_t s);

// -------------------------------------------------------------- SwiGLU gate
// hq, sh = per-row quantization of h = silu(a) * b for ab = [a | b] [M, 2F]
// (dtype abt, pitch ldab); F <= 16384.
cudaError_t launch_swiglu_quant(const void* ab, int abt, int64_t M, int64_t F, int64_t ldab,
                                int8_t* hq, int64_t ldh, float* sh, int32_t* st, cudaStream_t s);
// dab [M, 2F] (dtype dabt, contiguous) = [da | db] from ab and dh [M, F] (dht).
cudaError_t launch_swiglu_bwd(const void* ab, int abt, int64_t ldab, const void* dh, int dht,
                              int64_t M, int64_t F, void* dab, int dabt, cudaStream_t s);

// -------------------------------------------------------------- GEMM
// out[r, c] = ((float)acc[r,c] * row_scale[r]) * col_scale[c] + bias[c]
// (each factor optional), then an optional in-register block-Hadamard of
// width hb (0 or 2..128) along c; acc = int8 x int8 -> int32 on tcgen05.
struct GemmEpilogue {
  void* out = nullptr;
  int out_bf16 = 0;
  int64_t ldo = 0;
  const float* row_scale = nullptr;
  const float* col_scale = nullptr;
  const float* bias = nullptr;
  int hb = 0;
  float hc = 1.0f;
  // launch_gemm_bf16 only, bf16 output, no scales or bias, rows and cols
  // multiples of 16: the elementwise Newton-Schulz steps in the epilogue.
  // With ns_x set (bf16 [rows, cols], pitch ldo, the same as out; out may be
  // ns_x itself): out = bf16(ns_a * x + ns_c * acc), each operation rounded
  // once (ns_c = 1 multiplies exactly).  With ns_xt also set, the stored
  // values are written transposed into ns_xt ([cols, rows] bf16, pitch
  // ns_ldt elements), which must not be an operand of the product.  With
  // ns_mirror (a symmetric product run with upper_only): each strictly upper
  // tile's stored values are written transposed into its lower mirror tile
  // of out, so out comes back complete.
  const void* ns_x = nullptr;
  void* ns_xt = nullptr;
  int64_t ns_ldt = 0;
  float ns_a = 0.0f, ns_c = 1.0f;
  int ns_mirror = 0;
};

// A: rows x contraction, K-major ([rows][kc], pitch lda bytes) or MN-major
// ([kc][rows], pitch lda).  B likewise with `cols`.  rows, cols >= 1, kc >= 1.
cudaError_t launch_gemm_i8(const int8_t* A, bool a_mn, int64_t lda, const int8_t* B, bool b_mn,
                           int64_t ldb, int64_t rows, int64_t cols, int64_t kc,
                           const GemmEpilogue& ep, int32_t* status, cudaStream_t s);

// The same products for contractions longer than the int32-safe 131,071:
// splits of at most 130,944 write raw int32 partial sums to `parts`
// (splits * rows * cols int32, 16-byte aligned; parts_elems is its capacity,
// checked before any launch), then one pass
// sums them in int64 and applies ep (hb must be 0; cols % 16 == 0).  Input
// gradient (K-major x MN-major) and weight gradient (MN-major x MN-major).
// With min_splits > 1 the same path spreads an output of at most 128 rows
// (one tile row) over more SMs: small_output_splits() gives the count, at
// most QL_SMALL_OUTPUT_SPLITS, so the partial sums need at most that many
// rows x cols int32 copies.
#define QL_SMALL_OUTPUT_SPLITS 8
int contraction_splits(int64_t kc);
int small_output_splits(int64_t rows, int64_t cols, int64_t kc);
cudaError_t launch_gemm_i8_long(const int8_t* A, bool a_mn, int64_t lda, const int8_t* B, bool b_mn,
                                int64_t ldb, int64_t rows, int64_t cols, int64_t kc,
                                int32_t* parts, size_t parts_elems, const GemmEpilogue& ep,
                                int32_t* status, cudaStream_t s, int min_splits = 1);

// The same GEMM on bf16 operands (tcgen05 kind::f16, float32 accumulator):
// A [rows][kc] and B [cols][kc] both K-major bf16 with pitches lda, ldb
// elements; out = acc * row_scale * col_scale + bias as above, hb must be 0.
// upper_only (optional, in/out): for a product known to be symmetric, set
// it to ask for the upper 256 x 256 tiles only; it comes back true when only
// those were written (CTA-pair tiles on a square grid), false when all were.
cudaError_t launch_gemm_bf16(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t rows,
                             int64_t cols, int64_t kc, const GemmEpilogue& ep, int32_t* status,
                             cudaStream_t s, bool* upper_only = nullptr);

// -------------------------------------------------------------- update
struct UpdateConsts {
  int kind = 0;  // 0 SGD, 1 AdamW
  float lr = 0, a = 1, st = 0, rbc2 = 1, b1 = 0, b2 = 0, omb1 = 0, omb2 = 0, eps = 0;
  // AdamW constants that keep sqrt(v)*rbc2 + eps inside [2^-60, 2^60] for
  // every v in [2^-100, 2^100]: the range of the fast square-root and
  // division steps (set by finish()).
  int fast = 0;
  void finish() {
    fast = eps >= 0x1p-60f && eps <= 1.0f && rbc2 >= 1.0f && rbc2 <= 512.0f;
  }
};

cudaError_t launch_update_sr(int8_t* wq, float* sw, const float* grad, int64_t N, int64_t K,
                             const UpdateConsts& c, float* m, float* v, uint64_t seed,
                             uint64_t step, float* g, float* g_m, float* g_v, int32_t* status,
                             cudaStream_t s);

}  // namespace ql
