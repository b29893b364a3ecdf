// qlinear_api.cu - the extern "C" entry points declared in include/qlinear.h.
// Each validates its arguments on the host (returning before any launch, so
// no output is touched on error) and then launches the kernels of
// rowops.cu, gemm_i8.cu and update_sr.cu on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <algorithm>

#include "launch.h"
#include "../../include/qlinear.h"

namespace ql {

const DeviceInfo& device_info() {
  static DeviceInfo infos[64];
  static std::once_flag once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::call_once(once[dev], [dev] {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    infos[dev].sms = sms > 0 ? sms : 1;
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    infos[dev].smem_optin = optin > 0 ? optin : 48 * 1024;
  });
  return infos[dev];
}

namespace {
std::atomic<uint64_t> g_launches{0};
constexpr int kMaxTimed = 16;
thread_local cudaEvent_t t_before[kMaxTimed];
thread_local cudaEvent_t t_after[kMaxTimed];
thread_local int t_timed = 0;  // pairs set
thread_local int t_next = 0;   // next pair to use
}  // namespace

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

void gemm_timing_events(cudaEvent_t* before, cudaEvent_t* after) {
  if (t_next < t_timed) {
    *before = t_before[t_next];
    *after = t_after[t_next];
    ++t_next;
  } else {
    *before = nullptr;
    *after = nullptr;
  }
}

}  // namespace ql

namespace {

using ql::GemmEpilogue;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_dtype(int t) { return t == QL_F32 || t == QL_BF16; }

inline int64_t elem_size(int t) { return t == QL_BF16 ? 2 : 4; }

inline bool valid_block(int B) { return B == 0 || (B >= 2 && B <= 256 && (B & (B - 1)) == 0); }

// c = 1/sqrt(B) computed in float64 and rounded once to float32.
inline float hadamard_c(int B) { return B > 0 ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(B))) : 1.0f; }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? QL_OK : QL_ERR_CUDA; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace carve-up shared by the two backward calls.
struct WsLayout {
  size_t dyq, s1, colmax, s2, colsum, dxtmp, parts, parts_elems, total;
};

// Contractions longer than the int32-safe 131,071 (the input gradient's over
// N output classes, the weight gradient's over M tokens) run in splits whose
// int32 partial sums wait in `parts` to be combined in int64.
WsLayout ws_layout(int64_t M, int64_t N, int64_t K, int B) {
  WsLayout L;
  const size_t m = static_cast<size_t>(M), n = static_cast<size_t>(N), k = static_cast<size_t>(K);
  // Outputs of at most 128 rows (few tokens for dX, few output features for
  // dW) also run split, to spread over more SMs.
  size_t dx_splits = N > QL_MAX_CONTRACTION ? ql::contraction_splits(N) : 0;
  size_t dw_splits = M > QL_MAX_CONTRACTION ? ql::contraction_splits(M) : 0;
  if (M <= 128) dx_splits = std::max<size_t>(dx_splits, QL_SMALL_OUTPUT_SPLITS);
  if (N <= 128) dw_splits = std::max<size_t>(dw_splits, QL_SMALL_OUTPUT_SPLITS);
  size_t off = 0;
  L.dyq = off;    off += align256(m * n);
  L.s1 = off;     off += align256(4 * (M > 0 ? m : 1));
  L.colmax = off; off += align256(4 * (N > 0 ? n : 1));
  L.s2 = off;     off += align256(4 * (N > 0 ? n : 1));
  L.colsum = off; off += align256(8 * (N > 0 ? n : 1));
  L.dxtmp = off;
  if (B > 128 || (dx_splits > 0 && B > 0)) off += align256(4 * m * k);
  L.parts = off;
  L.parts_elems = std::max(dx_splits * m * k, dw_splits * n * k);
  off += align256(4 * L.parts_elems);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(base) + off);
}

// The input-gradient product from the row-quantized dY: dX = s1[m] *
// (dyq_r W_q), times R when B > 0 (fused into the GEMM epilogue for B <= 128;
// a second pass over a float32 product for B = 256 and for split contractions).
int run_dx_product(const int8_t* dyq_r, const int8_t* wq, const float* s1, int64_t M, int64_t N,
                   int64_t K, int B, void* dx, int dxt, void* ws, const WsLayout& L,
                   int32_t* status, cudaStream_t s) {
  GemmEpilogue ep;
  ep.row_scale = s1;
  ep.ldo = K;
  const int small = M <= 128 ? ql::small_output_splits(M, K, N) : 1;
  const bool split = N > QL_MAX_CONTRACTION || small > 1;
  int32_t* parts = at<int32_t>(ws, L.parts);
  if (B > 128 || (split && B > 0)) {
    float* tmp = dxt == QL_F32 ? reinterpret_cast<float*>(dx) : at<float>(ws, L.dxtmp);
    ep.out = tmp;
    cudaError_t e = split ? ql::launch_gemm_i8_long(dyq_r, false, N, wq, true, K, M, K, N, parts, L.parts_elems, ep, status, s, small)
                          : ql::launch_gemm_i8(dyq_r, false, N, wq, true, K, M, K, N, ep, status, s);
    if (e != cudaSuccess) return QL_ERR_CUDA;
    return cuda_status(ql::launch_hadamard(tmp, QL_F32, K, dx, dxt, K, M, K, B, hadamard_c(B), s));
  }
  ep.out = dx;
  ep.out_bf16 = dxt == QL_BF16;
  if (split)
    return cuda_status(ql::launch_gemm_i8_long(dyq_r, false, N, wq, true, K, M, K, N, parts, L.parts_elems, ep, status, s, small));
  ep.hb = B;
  ep.hc = hadamard_c(B);
  return cuda_status(ql::launch_gemm_i8(dyq_r, false, N, wq, true, K, M, K, N, ep, status, s));
}

// The weight-gradient product from the column-quantized dY: dW = s2[n] *
// (dyq_c^T X_q), the contraction over the M tokens.
int run_dw_product(const int8_t* dyq_c, const int8_t* xq, const float* s2, int64_t M, int64_t N,
                   int64_t K, float* dw, void* ws, const WsLayout& L, int32_t* status,
                   cudaStream_t s) {
  GemmEpilogue ep;
  ep.out = dw;
  ep.ldo = K;
  ep.row_scale = s2;
  const int small = N <= 128 ? ql::small_output_splits(N, K, M) : 1;
  if (M > QL_MAX_CONTRACTION || small > 1)
    return cuda_status(ql::launch_gemm_i8_long(dyq_c, true, N, xq, true, K, N, K, M,
                                               at<int32_t>(ws, L.parts), L.parts_elems, ep,
                                               status, s, small));
  return cuda_status(ql::launch_gemm_i8(dyq_c, true, N, xq, true, K, N, K, M, ep, status, s));
}

}  // namespace

namespace ql {

int check_bwd_dx_args(const void* dy, int dyt, int64_t M, int64_t N, const int8_t* wq,
                      const float* sw, int64_t K, int hadamard_block, const void* dx, int dxt,
                      const int32_t* d_status, bool* noop) {
  *noop = false;
  if (!valid_dtype(dyt) || !valid_dtype(dxt) || !valid_block(hadamard_block)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || M > INT32_MAX ||
      K > INT32_MAX)
    return QL_ERR_SHAPE;
  if (hadamard_block > 0 && K % hadamard_block != 0) return QL_ERR_SHAPE;
  if (M == 0 || K == 0) {
    *noop = true;
    return QL_OK;
  }
  if (!dx || !d_status || (N > 0 && (!dy || !wq || !sw))) return QL_ERR_ARG;
  return QL_OK;
}

}  // namespace ql

extern "C" {

void ql_set_gemm_timing_events(void* const* before, void* const* after, int n) {
  if (n < 0 || !before || !after) n = 0;
  if (n > ql::kMaxTimed) n = ql::kMaxTimed;
  for (int i = 0; i < n; ++i) {
    ql::t_before[i] = reinterpret_cast<cudaEvent_t>(before[i]);
    ql::t_after[i] = reinterpret_cast<cudaEvent_t>(after[i]);
  }
  ql::t_timed = n;
  ql::t_next = 0;
}

uint64_t ql_kernel_launches(void) { return ql::g_launches.load(std::memory_order_relaxed); }

const char* ql_status_string(int status) {
  switch (status) {
    case QL_OK: return "QL_OK";
    case QL_ERR_ARG: return "QL_ERR_ARG: invalid argument";
    case QL_ERR_SHAPE: return "QL_ERR_SHAPE: invalid shape, block size or workspace size";
    case QL_ERR_ALIGN: return "QL_ERR_ALIGN: pointer or pitch not 16-byte aligned";
    case QL_ERR_ZERO_ROW: return "QL_ERR_ZERO_ROW: rejected all-zero row";
    case QL_ERR_NONFINITE: return "QL_ERR_NONFINITE: inf or NaN in the input";
    case QL_ERR_UNSUPPORTED: return "QL_ERR_UNSUPPORTED: size beyond the supported range";
    case QL_ERR_CUDA: return "QL_ERR_CUDA: CUDA runtime error";
    case QL_ERR_TIMEOUT: return "QL_ERR_TIMEOUT: device wait timed out";
    default: return "unknown ql_status";
  }
}

size_t qlinear_workspace_bytes(int64_t M, int64_t N, int64_t K, int hadamard_block) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return ws_layout(M, N, K, hadamard_block).total;
}

int qlinear_quantize_rows(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                          const float* col_scale, int hadamard_block, unsigned flags, int8_t* q,
                          int64_t ldq, float* row_scale, int32_t* d_status, void* stream) {
  if (!valid_dtype(xt) || !valid_block(hadamard_block) || (flags & ~QL_REJECT_ZERO_ROWS))
    return QL_ERR_ARG;
  if (rows < 0 || cols < 0 || cols % 16 != 0 || ldx < cols || ldq < cols || ldq % 16 != 0 ||
      cols > INT32_MAX)
    return QL_ERR_SHAPE;
  if (hadamard_block > 0 && cols % hadamard_block != 0) return QL_ERR_SHAPE;
  if (rows == 0) return QL_OK;
  if (!x || !q || !row_scale || !d_status) return QL_ERR_ARG;
  if (!aligned16(x) || !aligned16(q) || (ldx * elem_size(xt)) % 16 != 0 ||
      (col_scale && !aligned16(col_scale)))
    return QL_ERR_ALIGN;
  return cuda_status(ql::launch_quant_rows(x, xt, rows, cols, ldx, col_scale, hadamard_block,
                                           hadamard_c(hadamard_block), flags, q, ldq, row_scale,
                                           d_status, as_stream(stream)));
}

int qlinear_hadamard(const void* x, int xt, int64_t ldx, void* y, int yt, int64_t ldy,
                     int64_t rows, int64_t cols, int hadamard_block, void* stream) {
  if (!valid_dtype(xt) || !valid_dtype(yt) || !valid_block(hadamard_block) || hadamard_block == 0)
    return QL_ERR_ARG;
  if (rows < 0 || cols < 0 || cols % 16 != 0 || cols % hadamard_block != 0 || ldx < cols ||
      ldy < cols || cols > INT32_MAX)
    return QL_ERR_SHAPE;
  if (rows == 0 || cols == 0) return QL_OK;
  if (!x || !y) return QL_ERR_ARG;
  if (x == y && (xt != yt || ldx != ldy)) return QL_ERR_ARG;
  if (!aligned16(x) || !aligned16(y) || (ldx * elem_size(xt)) % 16 != 0 ||
      (ldy * elem_size(yt)) % 16 != 0)
    return QL_ERR_ALIGN;
  return cuda_status(ql::launch_hadamard(x, xt, ldx, y, yt, ldy, rows, cols, hadamard_block,
                                         hadamard_c(hadamard_block), as_stream(stream)));
}

int qlinear_fwd(const void* x, int xt, int64_t M, int64_t K, const int8_t* wq, const float* sw,
                int64_t N, const float* bias, int hadamard_block, void* y, int yt,
                int8_t* xq_saved, float* sx_saved, int32_t* d_status, void* stream) {
  if (!valid_dtype(xt) || !valid_dtype(yt) || !valid_block(hadamard_block)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || M > INT32_MAX ||
      N > INT32_MAX)
    return QL_ERR_SHAPE;
  if (hadamard_block > 0 && K % hadamard_block != 0) return QL_ERR_SHAPE;
  if (K > QL_MAX_CONTRACTION) return QL_ERR_UNSUPPORTED;
  if (M == 0) return QL_OK;
  // With K == 0 the input, codes and weight are empty (possibly NULL).
  if (!sx_saved || !d_status || (K > 0 && (!x || !xq_saved)) ||
      (N > 0 && (!y || (K > 0 && (!wq || !sw)))))
    return QL_ERR_ARG;
  if ((K > 0 && (!aligned16(x) || !aligned16(xq_saved))) ||
      (N > 0 && (!aligned16(y) || (K > 0 && (!aligned16(wq) || !aligned16(sw))))) ||
      (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = ql::launch_quant_rows(x, xt, M, K, K, nullptr, hadamard_block,
                                        hadamard_c(hadamard_block), 0u, xq_saved, K, sx_saved,
                                        d_status, s);
  if (e != cudaSuccess || N == 0) return cuda_status(e);
  if (K == 0) return cuda_status(ql::launch_fill_rows(y, yt, M, N, bias, s));
  GemmEpilogue ep;
  ep.out = y;
  ep.out_bf16 = yt == QL_BF16;
  ep.ldo = N;
  ep.row_scale = sx_saved;
  ep.col_scale = sw;
  ep.bias = bias;
  return cuda_status(ql::launch_gemm_i8(xq_saved, false, K, wq, false, K, M, N, K, ep, d_status, s));
}

int qlinear_fwd_quantized(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                          const int8_t* wq, const float* sw, int64_t N, const float* bias, void* y,
                          int yt, int32_t* d_status, void* stream) {
  if (!valid_dtype(yt)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || M > INT32_MAX || N > INT32_MAX)
    return QL_ERR_SHAPE;
  if (K > QL_MAX_CONTRACTION) return QL_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return QL_OK;
  if (!y || !d_status || (K > 0 && (!xq || !sx || !wq || !sw))) return QL_ERR_ARG;
  if (!aligned16(y) || (bias && !aligned16(bias)) ||
      (K > 0 && (!aligned16(xq) || !aligned16(wq) || !aligned16(sw))))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (K == 0) return cuda_status(ql::launch_fill_rows(y, yt, M, N, bias, s));
  GemmEpilogue ep;
  ep.out = y;
  ep.out_bf16 = yt == QL_BF16;
  ep.ldo = N;
  ep.row_scale = sx;
  ep.col_scale = sw;
  ep.bias = bias;
  return cuda_status(ql::launch_gemm_i8(xq, false, K, wq, false, K, M, N, K, ep, d_status, s));
}

int qlinear_swiglu_quantize(const void* ab, int abt, int64_t M, int64_t F, int64_t ldab,
                            int8_t* hq, int64_t ldh, float* sh, int32_t* d_status, void* stream) {
  if (!valid_dtype(abt)) return QL_ERR_ARG;
  if (M < 0 || F < 16 || F % 16 != 0 || ldab < 2 * F || ldh < F || ldh % 16 != 0 ||
      M > INT32_MAX)
    return QL_ERR_SHAPE;
  if (F > 16384) return QL_ERR_UNSUPPORTED;
  if (M == 0) return QL_OK;
  if (!ab || !hq || !sh || !d_status) return QL_ERR_ARG;
  if (!aligned16(ab) || !aligned16(hq) || (ldab * elem_size(abt)) % 16 != 0) return QL_ERR_ALIGN;
  return cuda_status(ql::launch_swiglu_quant(ab, abt, M, F, ldab, hq, ldh, sh, d_status,
                                             as_stream(stream)));
}

int qlinear_swiglu_bwd(const void* ab, int abt, int64_t ldab, const void* dh, int dht, int64_t M,
                       int64_t F, void* dab, int dabt, void* stream) {
  if (!valid_dtype(abt) || !valid_dtype(dht) || !valid_dtype(dabt)) return QL_ERR_ARG;
  if (M < 0 || F < 16 || F % 16 != 0 || ldab < 2 * F || F > INT32_MAX / 2) return QL_ERR_SHAPE;
  if (M == 0) return QL_OK;
  if (!ab || !dh || !dab) return QL_ERR_ARG;
  if (!aligned16(ab) || !aligned16(dh) || !aligned16(dab) || (ldab * elem_size(abt)) % 16 != 0)
    return QL_ERR_ALIGN;
  return cuda_status(ql::launch_swiglu_bwd(ab, abt, ldab, dh, dht, M, F, dab, dabt,
                                           as_stream(stream)));
}

int qlinear_dequantize(const int8_t* wq, int64_t ldq, const float* sw, int64_t N, int64_t K,
                       int hadamard_block, void* w, int wt, int64_t ldw, void* stream) {
  if (!valid_dtype(wt) || !valid_block(hadamard_block)) return QL_ERR_ARG;
  if (N < 0 || K < 0 || K % 16 != 0 || N > INT32_MAX || K > INT32_MAX || ldq < K ||
      ldq % 16 != 0 || ldw < K || (hadamard_block > 0 && K % hadamard_block != 0))
    return QL_ERR_SHAPE;
  if (N == 0 || K == 0) return QL_OK;
  if (!wq || !sw || !w) return QL_ERR_ARG;
  if (!aligned16(wq) || !aligned16(w) || (ldw * elem_size(wt)) % 16 != 0) return QL_ERR_ALIGN;
  return cuda_status(ql::launch_dequant_rows(wq, ldq, sw, w, wt, ldw, N, K, hadamard_block,
                                             hadamard_c(hadamard_block), as_stream(stream)));
}

int qlinear_codes_bf16(const int8_t* wq, int64_t ldq, int64_t N, int64_t K, void* out,
                       int64_t ldo, void* stream) {
  if (N < 0 || K < 0 || K % 16 != 0 || N > INT32_MAX || K > INT32_MAX || ldq < K ||
      ldq % 16 != 0 || ldo < K)
    return QL_ERR_SHAPE;
  if (N == 0 || K == 0) return QL_OK;
  if (!wq || !out) return QL_ERR_ARG;
  if (!aligned16(wq) || !aligned16(out) || (ldo * 2) % 16 != 0) return QL_ERR_ALIGN;
  // The codes times 1.0 (exact) stored as bf16 (exact).
  return cuda_status(ql::launch_dequant_rows(wq, ldq, nullptr, out, QL_BF16, ldo, N, K, 0, 1.0f,
                                             as_stream(stream)));
}

size_t qlinear_fwd_bf16_workspace_bytes(int64_t M, int64_t K, int xt, int hadamard_block) {
  if (M < 0 || K < 0) return 0;
  if (xt == QL_BF16 && hadamard_block == 0) return 0;
  return align256(2 * static_cast<size_t>(M) * static_cast<size_t>(K));
}

int qlinear_fwd_bf16(const void* x, int xt, int64_t M, int64_t K, const void* wq_bf16,
                     const float* sw, int64_t N, const float* bias, int hadamard_block, void* y,
                     int yt, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (!valid_dtype(xt) || !valid_dtype(yt) || !valid_block(hadamard_block)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || M > INT32_MAX || N > INT32_MAX ||
      K > INT32_MAX || (hadamard_block > 0 && K % hadamard_block != 0))
    return QL_ERR_SHAPE;
  if (M == 0 || N == 0) return QL_OK;
  if (!y || !d_status || (K > 0 && (!x || !wq_bf16 || !sw))) return QL_ERR_ARG;
  const bool need_xr = K > 0 && !(xt == QL_BF16 && hadamard_block == 0);
  if (need_xr && (!ws || ws_bytes < qlinear_fwd_bf16_workspace_bytes(M, K, xt, hadamard_block)))
    return QL_ERR_SHAPE;
  if (!aligned16(y) || (bias && !aligned16(bias)) ||
      (K > 0 && (!aligned16(x) || !aligned16(wq_bf16) || !aligned16(sw))) ||
      (need_xr && (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (K == 0) return cuda_status(ql::launch_fill_rows(y, yt, M, N, bias, s));
  const void* xr = x;
  if (need_xr) {
    cudaError_t e = ql::launch_hadamard(x, xt, K, ws, QL_BF16, K, M, K, hadamard_block,
                                        hadamard_c(hadamard_block), s);
    if (e != cudaSuccess) return QL_ERR_CUDA;
    xr = ws;
  }
  GemmEpilogue ep;
  ep.out = y;
  ep.out_bf16 = yt == QL_BF16;
  ep.ldo = N;
  ep.col_scale = sw;
  ep.bias = bias;
  return cuda_status(ql::launch_gemm_bf16(xr, K, wq_bf16, K, M, N, K, ep, d_status, s));
}

int qlinear_bwd_dx(const void* dy, int dyt, int64_t M, int64_t N, const int8_t* wq,
                   const float* sw, int64_t K, int hadamard_block, void* dx, int dxt, void* ws,
                   size_t ws_bytes, int32_t* d_status, void* stream) {
  bool noop = false;
  const int pre = ql::check_bwd_dx_args(dy, dyt, M, N, wq, sw, K, hadamard_block, dx, dxt,
                                        d_status, &noop);
  if (pre != QL_OK || noop) return pre;
  const WsLayout L = ws_layout(M, N, K, hadamard_block);
  if (!ws) return QL_ERR_ARG;
  if (ws_bytes < L.total) return QL_ERR_SHAPE;
  if (!aligned16(dx) || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      (N > 0 && (!aligned16(dy) || !aligned16(wq) || !aligned16(sw))))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (N == 0) {  // empty contraction: dX = 0
    return cuda_status(cudaMemsetAsync(dx, 0, static_cast<size_t>(M * K * elem_size(dxt)), s));
  }
  int8_t* dyq = at<int8_t>(ws, L.dyq);
  float* s1 = at<float>(ws, L.s1);
  cudaError_t e = ql::launch_quant_rows(dy, dyt, M, N, N, sw, 0, 1.0f, 0u, dyq, N, s1, d_status, s);
  if (e != cudaSuccess) return QL_ERR_CUDA;
  return run_dx_product(dyq, wq, s1, M, N, K, hadamard_block, dx, dxt, ws, L, d_status, s);
}

int qlinear_bwd_dw(const void* dy, int dyt, int64_t M, int64_t N, const int8_t* xq,
                   const float* sx, int64_t K, float* dw, float* db, void* ws, size_t ws_bytes,
                   int32_t* d_status, void* stream) {
  if (!valid_dtype(dyt)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || N > INT32_MAX || K > INT32_MAX)
    return QL_ERR_SHAPE;
  if (N == 0) return QL_OK;
  const WsLayout L = ws_layout(M, N, K, 0);
  if (!d_status || !ws || (K > 0 && !dw) || (M > 0 && (!dy || !xq || !sx))) return QL_ERR_ARG;
  if (ws_bytes < L.total) return QL_ERR_SHAPE;
  if ((dw && !aligned16(dw)) || (db && !aligned16(db)) || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      (M > 0 && (!aligned16(dy) || !aligned16(xq) || !aligned16(sx))))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (M == 0) {  // empty contraction: dW = 0, db = 0
    if (K > 0 && cudaMemsetAsync(dw, 0, static_cast<size_t>(N * K) * 4, s) != cudaSuccess)
      return QL_ERR_CUDA;
    if (db && cudaMemsetAsync(db, 0, static_cast<size_t>(N) * 4, s) != cudaSuccess)
      return QL_ERR_CUDA;
    return QL_OK;
  }
  uint32_t* colmax = at<uint32_t>(ws, L.colmax);
  double* colsum = at<double>(ws, L.colsum);
  float* s2 = at<float>(ws, L.s2);
  int8_t* dyq = at<int8_t>(ws, L.dyq);
  if (ql::launch_zero_stats(colmax, colsum, N, nullptr, 0, s) != cudaSuccess) return QL_ERR_CUDA;
  cudaError_t e = ql::launch_colstats(dy, dyt, M, N, sx, colmax, colsum, nullptr, nullptr,
                                      d_status, s);
  if (e == cudaSuccess)
    e = ql::launch_dualquant(dy, dyt, M, N, nullptr, sx, colmax, colsum, nullptr, nullptr, s2, db,
                             nullptr, dyq, d_status, s);
  if (e != cudaSuccess || K == 0) return cuda_status(e);
  return run_dw_product(dyq, xq, s2, M, N, K, dw, ws, L, d_status, s);
}

// qlinear_bwd's workspace: the common layout, then the column-quantized
// codes [M*N] and the row maxima [M].
size_t bwd_extra(int64_t M, int64_t N) {
  return align256(static_cast<size_t>(M) * static_cast<size_t>(N)) +
         align256(4 * static_cast<size_t>(M > 0 ? M : 1));
}

size_t qlinear_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int hadamard_block) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return ws_layout(M, N, K, hadamard_block).total + bwd_extra(M, N);
}

int qlinear_bwd(const void* dy, int dyt, int64_t M, int64_t N, const int8_t* wq, const float* sw,
                const int8_t* xq, const float* sx, int64_t K, int hadamard_block, void* dx,
                int dxt, float* dw, float* db, void* ws, size_t ws_bytes, int32_t* d_status,
                void* stream) {
  if (!valid_dtype(dyt) || !valid_dtype(dxt) || !valid_block(hadamard_block)) return QL_ERR_ARG;
  if (M < 0 || K < 0 || N < 0 || K % 16 != 0 || N % 16 != 0 || M > INT32_MAX ||
      N > INT32_MAX || K > INT32_MAX)
    return QL_ERR_SHAPE;
  if (hadamard_block > 0 && K % hadamard_block != 0) return QL_ERR_SHAPE;
  const WsLayout L = ws_layout(M, N, K, hadamard_block);
  const size_t need = L.total + bwd_extra(M, N);
  if (!d_status || !ws) return QL_ERR_ARG;
  if (ws_bytes < need) return QL_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return QL_ERR_ALIGN;
  const bool fused = M > 0 && N > 0 && K > 0;
  if (!fused) {
    // Degenerate sizes: the two separate calls (stream-ordered, so they may
    // share the workspace).
    int r = qlinear_bwd_dx(dy, dyt, M, N, wq, sw, K, hadamard_block, dx, dxt, ws, ws_bytes,
                           d_status, stream);
    if (r != QL_OK) return r;
    return qlinear_bwd_dw(dy, dyt, M, N, xq, sx, K, dw, db, ws, ws_bytes, d_status, stream);
  }
  if (!dy || !wq || !sw || !xq || !sx || !dx || !dw) return QL_ERR_ARG;
  if (!aligned16(dy) || !aligned16(wq) || !aligned16(sw) || !aligned16(xq) || !aligned16(sx) ||
      !aligned16(dx) || !aligned16(dw) || (db && !aligned16(db)))
    return QL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  int8_t* dyq_r = at<int8_t>(ws, L.dyq);
  int8_t* dyq_c = at<int8_t>(ws, L.total);
  const size_t rm_off = L.total + align256(static_cast<size_t>(M) * static_cast<size_t>(N));
  uint32_t* rowmax = at<uint32_t>(ws, rm_off);
  float* s1 = at<float>(ws, L.s1);
  uint32_t* colmax = at<uint32_t>(ws, L.colmax);
  double* colsum = at<double>(ws, L.colsum);
  float* s2 = at<float>(ws, L.s2);
  // Pass 1 over dY: column maxima of |dY*s_x| and column sums, row maxima of
  // |dY*s_w|; pass 2: the scales and both code sets, elementwise.
  if (ql::launch_zero_stats(colmax, colsum, N, rowmax, M, s) != cudaSuccess) return QL_ERR_CUDA;
  cudaError_t e = ql::launch_colstats(dy, dyt, M, N, sx, colmax, colsum, sw, rowmax, d_status, s);
  if (e == cudaSuccess)
    e = ql::launch_dualquant(dy, dyt, M, N, sw, sx, colmax, colsum, rowmax, s1, s2, db, dyq_r,
                             dyq_c, d_status, s);
  if (e != cudaSuccess) return QL_ERR_CUDA;
  // Input gradient (as qlinear_bwd_dx after its quantization), then weight
  // gradient (as qlinear_bwd_dw after its quantization).
  const int r = run_dx_product(dyq_r, wq, s1, M, N, K, hadamard_block, dx, dxt, ws, L, d_status, s);
  if (r != QL_OK) return r;
  return run_dw_product(dyq_c, xq, s2, M, N, K, dw, ws, L, d_status, s);
}

size_t qweight_muon_workspace_bytes(int64_t N, int64_t K) {
  if (N < 0 || K < 0) return 0;
  return static_cast<size_t>(ql::muon_layout(N, K).total);
}

int qweight_muon_orthogonalize(const float* grad, float* mom, int64_t N, int64_t K, float momentum,
                               int ns_steps, void* O, void* ws, size_t ws_bytes,
                               int32_t* d_status, void* stream) {
  if (!(momentum >= 0.0f && momentum < 1.0f) || ns_steps < 1 || ns_steps > 16) return QL_ERR_ARG;
  if (N < 0 || K < 0 || N % 16 != 0 || K % 16 != 0 || N > INT32_MAX || K > INT32_MAX)
    return QL_ERR_SHAPE;
  if (N == 0 || K == 0) return QL_OK;
  if (!grad || !mom || !O || !ws || !d_status) return QL_ERR_ARG;
  if (ws_bytes < qweight_muon_workspace_bytes(N, K)) return QL_ERR_SHAPE;
  if (!aligned16(grad) || !aligned16(mom) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return QL_ERR_ALIGN;
  return cuda_status(ql::launch_muon_orthogonalize(grad, mom, N, K, momentum, ns_steps, O, ws,
                                                   d_status, as_stream(stream)));
}

int qweight_update_muon_sr(int8_t* wq, float* sw, const void* O, int64_t N, int64_t K, float lr,
                           float weight_decay, uint64_t seed, uint64_t step, int32_t* d_status,
                           void* stream) {
  if (!std::isfinite(lr) || !std::isfinite(weight_decay) || step < 1) return QL_ERR_ARG;
  if (N < 0 || K < 0 || N % 16 != 0 || K % 16 != 0 || N > INT32_MAX) return QL_ERR_SHAPE;
  if (K > 32768) return QL_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return QL_OK;
  if (!wq || !sw || !O || !d_status) return QL_ERR_ARG;
  if (!aligned16(wq) || !aligned16(O)) return QL_ERR_ALIGN;
  // Host constants in float64, each rounded once: the decoupled decay factor
  // and the step size times max(1, N/K)^0.5.
  const double scale = N > K ? std::sqrt(static_cast<double>(N) / static_cast<double>(K)) : 1.0;
  const float a = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  const float st = static_cast<float>(static_cast<double>(lr) * scale);
  return cuda_status(ql::launch_update_dir(wq, sw, O, N, K, a, st, seed, step, d_status,
                                           as_stream(stream)));
}

int qvector_adamw(float* p, const float* g, float* m, float* v, int64_t n, const ql_optim* opt,
                  uint64_t step, int32_t* d_status, void* stream) {
  if (!opt || opt->kind != QL_ADAMW || step < 1 || !std::isfinite(opt->lr) ||
      !(opt->beta1 >= 0.0f && opt->beta1 < 1.0f) || !(opt->beta2 >= 0.0f && opt->beta2 < 1.0f) ||
      !std::isfinite(opt->eps) || !std::isfinite(opt->weight_decay))
    return QL_ERR_ARG;
  if (n < 0) return QL_ERR_SHAPE;
  if (n == 0) return QL_OK;
  if (!p || !g || !m || !v || !d_status) return QL_ERR_ARG;
  ql::UpdateConsts c;
  c.kind = QL_ADAMW;
  c.lr = opt->lr;
  const double t = static_cast<double>(step);
  c.a = static_cast<float>(1.0 - static_cast<double>(opt->lr) * static_cast<double>(opt->weight_decay));
  c.st = static_cast<float>(static_cast<double>(opt->lr) / (1.0 - std::pow(static_cast<double>(opt->beta1), t)));
  c.rbc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(opt->beta2), t)));
  c.b1 = opt->beta1;
  c.b2 = opt->beta2;
  c.omb1 = static_cast<float>(1.0 - static_cast<double>(opt->beta1));
  c.omb2 = static_cast<float>(1.0 - static_cast<double>(opt->beta2));
  c.eps = opt->eps;
  c.finish();
  return cuda_status(ql::launch_adamw_vector(p, g, m, v, n, c, d_status, as_stream(stream)));
}

int qweight_update_sr(int8_t* wq, float* sw, const float* grad, int64_t N, int64_t K,
                      const ql_optim* opt, float* m, float* v, uint64_t seed, uint64_t step,
                      const ql_weightnorm* wn, int32_t* d_status, void* stream) {
  if (!opt || (opt->kind != QL_SGD && opt->kind != QL_ADAMW) || step < 1) return QL_ERR_ARG;
  if (opt->kind == QL_SGD && opt->weight_decay != 0.0f) return QL_ERR_ARG;
  if (!std::isfinite(opt->lr) || (opt->kind == QL_ADAMW &&
                                  (!(opt->beta1 >= 0.0f && opt->beta1 < 1.0f) ||
                                   !(opt->beta2 >= 0.0f && opt->beta2 < 1.0f) ||
                                   !std::isfinite(opt->eps) || !std::isfinite(opt->weight_decay))))
    return QL_ERR_ARG;
  if (N < 0 || K < 0 || K % 16 != 0 || N > INT32_MAX) return QL_ERR_SHAPE;
  if (K > 32768) return QL_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return QL_OK;
  if (!wq || !sw || !grad || !d_status) return QL_ERR_ARG;
  if (opt->kind == QL_ADAMW && (!m || !v)) return QL_ERR_ARG;
  if (wn && (!wn->g || (opt->kind == QL_ADAMW && (!wn->g_m || !wn->g_v)))) return QL_ERR_ARG;
  if (!aligned16(wq) || !aligned16(grad) || (m && !aligned16(m)) || (v && !aligned16(v)))
    return QL_ERR_ALIGN;
  ql::UpdateConsts c;
  c.kind = opt->kind;
  c.lr = opt->lr;
  if (opt->kind == QL_ADAMW) {
    // Host constants, each computed in float64 and rounded once.
    const double t = static_cast<double>(step);
    c.a = static_cast<float>(1.0 - static_cast<double>(opt->lr) * static_cast<double>(opt->weight_decay));
    c.st = static_cast<float>(static_cast<double>(opt->lr) / (1.0 - std::pow(static_cast<double>(opt->beta1), t)));
    c.rbc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(opt->beta2), t)));
    c.b1 = opt->beta1;
    c.b2 = opt->beta2;
    c.omb1 = static_cast<float>(1.0 - static_cast<double>(opt->beta1));
    c.omb2 = static_cast<float>(1.0 - static_cast<double>(opt->beta2));
    c.eps = opt->eps;
    c.finish();
  }
  return cuda_status(ql::launch_update_sr(wq, sw, grad, N, K, c, m, v, seed, step,
                                          wn ? wn->g : nullptr, wn ? wn->g_m : nullptr,
                                          wn ? wn->g_v : nullptr, d_status, as_stream(stream)));
}

}  // extern "C"
