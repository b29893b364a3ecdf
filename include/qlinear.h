/*
 * qlinear.h - C ABI of the INT8 quantized-training Linear layer for NVIDIA
 * B200 (sm_100a).
 *
 * The layer keeps its weight as int8 codes with one float32 scale per output
 * row and no floating master copy; it quantizes its input per row on every
 * call, saves the int8 input for backward, runs int8 x int8 -> int32 GEMMs on
 * the tensor cores for the forward and both backward products, and updates
 * the weight with a stochastic requantization after each optimizer step.  An
 * optional block-Hadamard rotation R along the contraction dimension spreads
 * channel outliers before quantization.  Sources, cited by page title and part:
 *
 *   [QT] mini_trainer "docs/quantized-training.md": intro paragraph (INT8
 *        weights and saved Linear inputs, integer forward/backward products,
 *        no floating master weight, biases/gradients/optimizer state stay
 *        float), feature table (row-wise weight norm with int8 direction and
 *        float magnitude, zero directions rejected; bias, batched,
 *        single-sample inputs; SGD and AdamW), the paragraph after the table
 *        (updates requantize stochastically, fused row kernels), and the
 *        paragraph on contractions above 131,071.
 *   [CR] OneTrainer PR #1681 "Int8 conv rot": opening summary (block-Hadamard
 *        rotation), commit note item 1 (activations quantized per row every
 *        call; int8 route vs bf16 route), item 2 ((xR)(WR)^T = xW^T: rotate x,
 *        never un-rotate W), item 3 (the torch._int_mm row floor, which this
 *        library does not have), closing Summary.
 *
 * Conventions for every entry point
 *   - Matrices are row-major.  M = tokens (rows of x), K = in_features,
 *     N = out_features.  All pointers are DEVICE pointers unless stated.
 *   - The caller owns every buffer.  The library never allocates device
 *     memory; its only global state is a per-device, one-time set-up on
 *     first use (kernel attributes, occupancy figures), kept in atomics:
 *     calls from several host threads are safe (two first calls may both
 *     run the set-up, which writes the same values).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on `stream` and never
 *     synchronizes.
 *   - Argument, shape and alignment errors are detected on the host before
 *     any launch and returned; no output is touched then.  Conditions found
 *     on the device (zero rows, non-finite values, a wait that timed out)
 *     are OR-ed as bits (1u << code) into *d_status, a caller-owned device
 *     int32 that the caller zeroes and reads after its own synchronization.
 *   - int8 operands and outputs need 16-byte aligned pointers and row pitches
 *     that are multiples of 16 bytes (the tensor-memory-access engine reads
 *     them); this is why K and N must be multiples of 16.  M has no floor:
 *     M = 1 is valid, unlike torch._int_mm's "more than 16 rows" ([CR] item 3).
 *   - Float inputs (x, dY) are float32 or bf16 (ql_dtype), 16-byte aligned.
 *   - The float arithmetic that decides an integer code is IEEE binary32
 *     with round-to-nearest-even and no fused multiply-add, so int8 codes,
 *     scales and stochastic-rounding results are reproducible bit for bit.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes.  Device-side conditions use the bit (1u << code). */
typedef enum {
    QL_OK = 0,
    QL_ERR_ARG = 1,         /* null pointer, bad enum, bad hyper-parameter      */
    QL_ERR_SHAPE = 2,       /* negative size, K or N not a multiple of 16,
                               bad Hadamard block, too-small workspace          */
    QL_ERR_ALIGN = 3,       /* pointer or row pitch not 16-byte aligned        */
    QL_ERR_ZERO_ROW = 4,    /* device: a rejected all-zero row / direction      */
    QL_ERR_NONFINITE = 5,   /* device: inf or NaN met; affected outputs are
                               unspecified                                       */
    QL_ERR_UNSUPPORTED = 6, /* forward K above 131,071 ([QT]), row too long     */
    QL_ERR_CUDA = 7,        /* a CUDA runtime call or launch failed              */
    QL_ERR_TIMEOUT = 8      /* device: a pipeline wait gave up (bounded waits;
                               the kernel returns instead of hanging)            */
} ql_status;

typedef enum { QL_F32 = 0, QL_BF16 = 1 } ql_dtype;

typedef enum { QL_SGD = 0, QL_ADAMW = 1 } ql_optim_kind;

/* Optimizer hyper-parameters.  SGD: w' = w - lr*g (no momentum; weight_decay
 * must be 0).  AdamW (decoupled weight decay): w1 = w*(1-lr*wd);
 * m' = b1*m + (1-b1)*g; v' = b2*v + (1-b2)*g*g;
 * w' = w1 - (lr/(1-b1^t)) * m' / (sqrt(v') * (1/sqrt(1-b2^t)) + eps), the
 * factors lr/(1-b1^t), 1/sqrt(1-b2^t), 1-lr*wd, 1-b1, 1-b2 each computed in
 * float64 on the host and rounded once to float32. */
typedef struct {
    int kind; /* ql_optim_kind */
    float lr, beta1, beta2, eps, weight_decay;
} ql_optim;

/* Row-wise weight normalization (dim=0, [QT] feature table): the stored int8
 * row is the direction v = s*q; the effective weight row is g[n]*q/||q||.
 * g is float32 [N]; g_m, g_v are its AdamW moments (may be NULL for SGD). */
typedef struct {
    float *g;
    float *g_m;
    float *g_v;
} ql_weightnorm;

/* qlinear_quantize_rows flag: report all-zero rows as QL_ERR_ZERO_ROW (used
 * when preparing weights: a zero direction cannot be represented). */
#define QL_REJECT_ZERO_ROWS 1u

/* Longest int32-safe contraction: no int8 dot product of this length can
 * leave int32, floor((2^31-1)/128^2) ([QT], contraction paragraph).  The
 * forward accepts contractions (K) up to it.  The backward products go past
 * it: the input gradient's sum over N output classes and the weight
 * gradient's sum over M tokens then run in splits of at most 130,944 whose
 * int32 partial sums are combined in int64 before scaling, exactly the int64
 * sum ([QT]: this keeps input gradients at large output-class counts from
 * saturating); the workspace grows by the partial sums. */
#define QL_MAX_CONTRACTION 131071

/* Human-readable name of a status code (static string). */
QL_API const char *ql_status_string(int status);

/* Bytes of device workspace that qlinear_bwd_dx / qlinear_bwd_dw need for
 * a layer of these sizes and Hadamard block (0 = no rotation).  The buffer is
 * scratch: its contents on entry do not matter and on exit are unspecified. */
QL_API size_t qlinear_workspace_bytes(int64_t M, int64_t N, int64_t K, int hadamard_block);

/* Per-row symmetric int8 quantization, optionally rotated ([CR] item 1 and
 * summary).  For each row r of x [rows, cols] (pitch ldx elements, dtype xt):
 *   t = x[r,:] * col_scale (elementwise, if col_scale != NULL)
 *   t = t R                (if hadamard_block = B > 0; R = blockdiag(H_B)/sqrt(B),
 *                           Sylvester order, butterflies h = 1..B/2 then one
 *                           multiply by fl32(1/sqrt(B)))
 *   amax = max|t|; row_scale[r] = amax/127; q[r,:] = clamp(rne(t*(127/amax)), +-127)
 * amax = 0 gives scale 0 and zero codes, and sets QL_ERR_ZERO_ROW in
 * *d_status when flags has QL_REJECT_ZERO_ROWS.  This is also the weight
 * preparation step: quantize W [N,K] with the layer's block and the flag.
 * Requirements: cols % 16 == 0; B in {0, 2, 4, ..., 256} with cols % B == 0;
 * ldx >= cols, ldq >= cols, ldq % 16 == 0; x, q 16-byte aligned and
 * ldx * sizeof(xt) % 16 == 0; col_scale (optional) 16-byte aligned. */
QL_API int qlinear_quantize_rows(const void *x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                          const float *col_scale, int hadamard_block, unsigned flags,
                          int8_t *q, int64_t ldq, float *row_scale,
                          int32_t *d_status, void *stream);

/* y = x R row by row (R as above), x [rows, cols] of dtype xt with pitch ldx,
 * y of dtype yt with pitch ldy; y == x (same dtype and pitch) is allowed.
 * R is its own inverse, so this also un-rotates (the "unquantized weight"
 * of [CR] item 2: dequantize the codes, then call this). */
QL_API int qlinear_hadamard(const void *x, int xt, int64_t ldx, void *y, int yt, int64_t ldy,
                     int64_t rows, int64_t cols, int hadamard_block, void *stream);

/* The weight back in floating point and in the original basis: the
 * "unquantized weight" that LoRA decomposition and offload sizing read
 * ([CR] third commit note, item 2: it un-rotates, only the forward uses the
 * stored rotated basis).  For each row n of the codes wq [N, K] (pitch ldq):
 *   w[n,:] = s_w[n] * wq[n,:]   (one float32 multiply per element)
 *   w[n,:] = w[n,:] R           (if hadamard_block = B > 0; R as above, its
 *                                own inverse, so this undoes the rotation
 *                                the weight preparation applied)
 * w [N, K] of dtype wt with pitch ldw (elements).  Requirements: K % 16 == 0,
 * B in {0, 2, ..., 256} with K % B == 0, ldq >= K and ldq % 16 == 0, ldw >= K,
 * wq and w 16-byte aligned, ldw * sizeof(wt) % 16 == 0.  Asynchronous on
 * `stream`; argument errors are returned before any launch. */
QL_API int qlinear_dequantize(const int8_t *wq, int64_t ldq, const float *sw, int64_t N,
                              int64_t K, int hadamard_block, void *w, int wt, int64_t ldw,
                              void *stream);

/* The codes of an int8 weight as bf16, exactly (|q| <= 127 needs 7
 * significant bits): the weight operand of qlinear_fwd_bf16, refreshed by
 * the caller after each update.  out [N, K] bf16 with pitch ldo elements;
 * same requirements as qlinear_dequantize. */
QL_API int qlinear_codes_bf16(const int8_t *wq, int64_t ldq, int64_t N, int64_t K, void *out,
                              int64_t ldo, void *stream);

/* The forward's bf16 route ([CR] third commit note, items 1 and 2): the
 * activations are rotated instead of the weight being un-rotated, and they
 * are not quantized.
 *   xr = bf16(x R)       (float32 butterflies as in qlinear_hadamard, one
 *                         rounding to bf16; with B = 0 just bf16(x), and x
 *                         itself when it is already bf16)
 *   y[m,n] = (sum_k xr[m,k] * q[n,k]) * s_w[n] + bias[n]
 * with the sum on the tensor cores (tcgen05 kind::f16, bf16 x bf16, float32
 * accumulator): x times the dequantized weight, transposed, up to rounding.
 * wq_bf16 [N, K]: the weight codes as bf16 (qlinear_codes_bf16), in the
 * weight's stored (rotated) basis; sw, bias as in qlinear_fwd.  y [M, N] of
 * dtype yt.  ws: qlinear_fwd_bf16_workspace_bytes(M, K, xt, B) bytes,
 * 256-byte aligned (holds xr; 0 bytes and NULL allowed when x is bf16 and
 * B = 0).  Requirements: K % 16 == 0, N % 16 == 0, B in {0, 2, ..., 256} with
 * K % B == 0; x, wq_bf16, y 16-byte aligned; contiguous rows.  No
 * contraction limit (float32 accumulation).  Device conditions (a bounded
 * wait that timed out) are OR-ed into *d_status. */
QL_API size_t qlinear_fwd_bf16_workspace_bytes(int64_t M, int64_t K, int xt, int hadamard_block);
QL_API int qlinear_fwd_bf16(const void *x, int xt, int64_t M, int64_t K, const void *wq_bf16,
                            const float *sw, int64_t N, const float *bias, int hadamard_block,
                            void *y, int yt, void *ws, size_t ws_bytes, int32_t *d_status,
                            void *stream);

/* Forward ([CR] item 1 and summary; [QT] intro):
 *   X_q, s_x = quantize_rows(x, B)                     (saved for backward)
 *   y[m,n] = ((float)(sum_k X_q[m,k] W_q[n,k]) * s_x[m]) * s_w[n] + bias[n]
 * x [M,K] (xt), W_q [N,K] int8 prepared in the same rotated basis, s_w [N],
 * bias [N] float32 or NULL, y [M,N] of dtype yt, xq_saved [M,K] int8,
 * sx_saved [M] float32.  K, N multiples of 16; K <= QL_MAX_CONTRACTION. */
QL_API int qlinear_fwd(const void *x, int xt, int64_t M, int64_t K,
                const int8_t *wq, const float *sw, int64_t N, const float *bias,
                int hadamard_block, void *y, int yt,
                int8_t *xq_saved, float *sx_saved, int32_t *d_status, void *stream);

/* Forward from an input that is already quantized: the GEMM and epilogue of
 * qlinear_fwd without its quantization step,
 *   y[m,n] = ((float)(sum_k xq[m,k] W_q[n,k]) * sx[m]) * s_w[n] + bias[n]
 * for codes xq [M,K] and row scales sx [M] that a producer kernel wrote in the
 * layer's own format (per-row symmetric int8, in the weight's basis), such as
 * qlinear_swiglu_quantize.  Sizes, layouts, requirements and errors as for
 * qlinear_fwd. */
QL_API int qlinear_fwd_quantized(const int8_t *xq, const float *sx, int64_t M, int64_t K,
                                 const int8_t *wq, const float *sw, int64_t N, const float *bias,
                                 void *y, int yt, int32_t *d_status, void *stream);

/* The SwiGLU gate of an MLP whose three projections are layers of this
 * library (w1 and w3 stacked as one [2F, d] weight on the same input, w2 on
 * h), fused with the per-row quantization that the second projection applies
 * to its input ([CR] item 1: activations quantized per row on every call), so
 * h never goes to memory:
 *   h[m,f] = silu(a[m,f]) * b[m,f],  silu(a) = a / (1 + e^-a)
 *   sh[m] = max_f |h[m,f]| / 127,  hq[m,f] = clamp(rne(h * (127/max|h|)), +-127)
 * with ab = [a | b] [M, 2F] (dtype abt, pitch ldab elements: a = columns
 * 0..F-1, b = columns F..2F-1), hq [M, F] int8 (pitch ldh), sh [M] float32.
 * All float32, one rounding per operation in the order written; e^x by fixed
 * float32 steps (Cody-Waite reduction with C1 = fl32(ln 2), degree-7 Taylor
 * series, fused multiply-adds), so codes are reproducible bit for bit.  A zero
 * row gives sh = 0 and zero codes; a non-finite h sets QL_ERR_NONFINITE.
 * The result is the input (xq, sx) of qlinear_fwd_quantized and the saved
 * input of the second projection's backward.  Requirements: F % 16 == 0,
 * 16 <= F <= 16384 (QL_ERR_UNSUPPORTED above), ldab >= 2F with ldab *
 * sizeof(abt) % 16 == 0, ldh >= F, ldh % 16 == 0; ab, hq 16-byte aligned. */
QL_API int qlinear_swiglu_quantize(const void *ab, int abt, int64_t M, int64_t F, int64_t ldab,
                                   int8_t *hq, int64_t ldh, float *sh, int32_t *d_status,
                                   void *stream);

/* The gate's backward: from dh [M, F] (dtype dht, contiguous; the input
 * gradient of the second projection) and ab as above, the gradient at the
 * stacked pre-activations dab [M, 2F] (dtype dabt, contiguous):
 *   d = 1 + e^-a, sigma = 1/d, silu = a/d
 *   da = (dh * b) * (sigma * (1 + a * (1 - sigma))),   db = dh * silu
 * float32, one rounding per operation in the order written (bf16 output:
 * the float32 value rounded to nearest even).  dab is the output gradient of
 * the stacked first projection.  Requirements: F % 16 == 0, F >= 16,
 * ldab >= 2F with ldab * sizeof(abt) % 16 == 0; ab, dh, dab 16-byte aligned. */
QL_API int qlinear_swiglu_bwd(const void *ab, int abt, int64_t ldab, const void *dh, int dht,
                              int64_t M, int64_t F, void *dab, int dabt, void *stream);

/* Input gradient ([QT] intro: the backward products are integer GEMMs too;
 * [CR] item 2 for the rotation):
 *   dYq, s' = quantize_rows(dY, col_scale = s_w)       (row quantization of dY*s_w)
 *   dX[m,k] = (float)(sum_n dYq[m,n] W_q[n,k]) * s'[m], then dX R if B > 0
 * (the layer saw xR, and R is symmetric, so dL/dx = dL/d(xR) R^T = (...) R).
 * dY [M,N] (dyt), W_q [N,K], s_w [N], dX [M,K] (dxt).  ws: device workspace of
 * at least qlinear_workspace_bytes(M,N,K,B) bytes, 256-byte aligned.
 * N above QL_MAX_CONTRACTION runs as int64-combined splits (see there). */
QL_API int qlinear_bwd_dx(const void *dy, int dyt, int64_t M, int64_t N,
                   const int8_t *wq, const float *sw, int64_t K, int hadamard_block,
                   void *dx, int dxt, void *ws, size_t ws_bytes,
                   int32_t *d_status, void *stream);

/* Weight (and bias) gradient from the int8-saved input ([QT] intro: the
 * Linear input is saved as int8 and the weight gradient is an integer GEMM;
 * biases and gradients stay float):
 *   t''[m,n] = dY[m,n]*s_x[m]; per column n: s''[n] = max_m|t''|/127,
 *   dYq_c[m,n] = clamp(rne(t''*(127/max_m|t''|)), +-127)
 *   dW[n,k] = (float)(sum_m dYq_c[m,n] X_q[m,k]) * s''[n]   (float32 [N,K],
 *             in the rotated basis when the layer is rotated)
 *   db[n]   = sum_m dY[m,n] (float64 sum rounded to float32), if db != NULL.
 * dY [M,N] (dyt), X_q [M,K] int8 and s_x [M] as saved by qlinear_fwd.
 * M above QL_MAX_CONTRACTION runs as int64-combined splits.  ws as for
 * qlinear_bwd_dx. */
QL_API int qlinear_bwd_dw(const void *dy, int dyt, int64_t M, int64_t N,
                   const int8_t *xq, const float *sx, int64_t K,
                   float *dw, float *db, void *ws, size_t ws_bytes,
                   int32_t *d_status, void *stream);

/* Bytes of device workspace that qlinear_bwd needs (qlinear_workspace_bytes
 * plus room for the second int8 copy of the gradient, M*N bytes). */
QL_API size_t qlinear_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int hadamard_block);

/* Both backward products of the layer in one call: exactly the results of
 * qlinear_bwd_dx (dX) followed by qlinear_bwd_dw (dW, db), but dY is read
 * twice instead of three times: one pass gathers the column maxima and sums,
 * a second pass writes both the row-quantized (dY*s_w) and the column-
 * quantized (dY*s_x) int8 copies from the same read.  Arguments as for the
 * two calls; ws holds qlinear_bwd_workspace_bytes(M, N, K, hadamard_block)
 * bytes.  Long contractions as for the two calls. */
QL_API int qlinear_bwd(const void *dy, int dyt, int64_t M, int64_t N,
                       const int8_t *wq, const float *sw, const int8_t *xq, const float *sx,
                       int64_t K, int hadamard_block, void *dx, int dxt, float *dw, float *db,
                       void *ws, size_t ws_bytes, int32_t *d_status, void *stream);

/* One optimizer step of an int8 weight [N,K] with stochastic requantization,
 * in place ([QT] paragraph after the feature table; rows "Optimizers",
 * "Row-wise weight normalization"):
 *   w = s_w[n]*q[n,k]; w' = step(w, grad) (SGD or AdamW, moments m, v float32
 *   [N,K] updated in place; NULL for SGD); per row: s' = max|w'|/127 and
 *   q'[n,k] = floor(w'*127/max|w'|) + 1 with probability equal to the
 *   fractional part, decided by u24 < frac*2^24 where u24 is the top 24 bits
 *   of word (e & 3) of Philox4x32-10 with key = seed and counter =
 *   (e>>2 low, e>>2 high, step low, step high), e = n*K + k.
 * With wn != NULL the rows are weight-norm directions: grad is the gradient
 * of the effective row g*q/||q||; the direction gradient
 *   dv = (g/(s*||q||)) * (grad - dg*q/||q||),  dg = sum_k grad*q/||q||
 * (dg summed in a fixed order: groups of 16 consecutive elements dealt
 * round-robin to 256 lanes, each lane in increasing k, then an xor butterfly
 * over the lanes with offsets 128..1) steps v = s*q, dg steps g; a zero
 * direction sets QL_ERR_ZERO_ROW and leaves its row and state unchanged.
 * opt and wn are HOST pointers (wn's members are device pointers).
 * step >= 1.  K % 16 == 0, K <= 32768. */
QL_API int qweight_update_sr(int8_t *wq, float *sw, const float *grad, int64_t N, int64_t K,
                      const ql_optim *opt, float *m, float *v,
                      uint64_t seed, uint64_t step, const ql_weightnorm *wn,
                      int32_t *d_status, void *stream);

/* MuonAuxAdamW ([QT] feature table, row "Optimizers", names it among the
 * update paths).  The pages do not define it; this follows the published
 * Muon optimizer (K. Jordan et al., "Muon: An optimizer for hidden layers in
 * neural networks", 2024) for the int8 weights, and AdamW (qvector_adamw)
 * for the float parameters such as biases.  One Muon step of a weight is
 * qweight_muon_orthogonalize followed by qweight_update_muon_sr.
 *
 * qweight_muon_orthogonalize: from the weight gradient grad [N, K] float32
 * and the momentum mom [N, K] float32 (updated in place):
 *   M' = beta*M + (1-beta)*G,  U = (1-beta)*G + beta*M'   (float32, in order)
 *   X = U, or U^T when N > K; X = X / (||X||_F + 1e-7)      (norm in float64)
 *   ns_steps times: A = X X^T;  B = b*A + c*(A A);  X = a*X + B X,
 *   (a, b, c) = (3.4445, -4.7750, 2.0315)
 * and O [N, K] bf16 = X in the weight's layout.  As in the published method
 * the products take bf16 operands (X, A and B rounded to bf16; float32
 * accumulation on the tensor cores), so O matches the float64 iteration of
 * the same definition to bf16 accuracy, not bit for bit.  ws: at least
 * qweight_muon_workspace_bytes(N, K) bytes, 256-byte aligned (for N = 7168,
 * K = 5376 about 0.35 GB).  Requirements: N, K multiples of 16; 0 <= beta < 1;
 * 1 <= ns_steps <= 16; grad, mom, O 16-byte aligned. */
QL_API size_t qweight_muon_workspace_bytes(int64_t N, int64_t K);
QL_API int qweight_muon_orthogonalize(const float *grad, float *mom, int64_t N, int64_t K,
                                      float momentum, int ns_steps, void *O, void *ws,
                                      size_t ws_bytes, int32_t *d_status, void *stream);

/* qweight_update_muon_sr: the Muon step of the int8 weight from O (bf16
 * [N, K]), in place, with the layer's stochastic requantization:
 *   w = s_w[n]*q;  w' = w*a - st*O,  a = fl32(1 - lr*wd),
 *   st = fl32(lr * max(1, N/K)^0.5)   (constants in float64, rounded once)
 * then per row s' = max|w'|/127 and codes by the Philox-keyed stochastic
 * rounding of qweight_update_sr (same seed/step/element keying).  Bit for
 * bit reproducible given O.  Requirements: N, K multiples of 16, K <= 32768,
 * step >= 1; wq, O 16-byte aligned. */
QL_API int qweight_update_muon_sr(int8_t *wq, float *sw, const void *O, int64_t N, int64_t K,
                                  float lr, float weight_decay, uint64_t seed, uint64_t step,
                                  int32_t *d_status, void *stream);

/* qvector_adamw: AdamW on a float32 vector p [n] with gradient g and moments
 * m, v (updated in place), the same per-element arithmetic and host
 * constants as qweight_update_sr's AdamW, without requantization (the
 * "AdamW" part of MuonAuxAdamW: biases and other float parameters).  opt is
 * a HOST pointer with kind QL_ADAMW; step >= 1.  A non-finite result sets
 * QL_ERR_NONFINITE. */
QL_API int qvector_adamw(float *p, const float *g, float *m, float *v, int64_t n,
                         const ql_optim *opt, uint64_t step, int32_t *d_status, void *stream);

/* Capacity of the library-owned scratch used by qlinear_bwd_dx_noalloc:
 * 32 MiB of device memory. */
#define QL_NOALLOC_SCRATCH_BYTES (32u << 20)

/* qlinear_bwd_dx_noalloc - the input gradient of qlinear_bwd_dx, for callers
 * that cannot allocate device memory and so cannot supply the `ws` buffer:
 * code running inside a host framework that owns all device memory and
 * forbids allocation while its kernels execute, or a process whose device
 * memory is fully reserved by another allocator.  (This entry point is an
 * interface convenience; the pages have no counterpart.)
 *
 * Arguments, results and errors are those of qlinear_bwd_dx without ws and
 * ws_bytes: its argument, shape and null-pointer checks come first and return
 * the same codes.  Instead of a caller buffer it uses a scratch array of
 * QL_NOALLOC_SCRATCH_BYTES that lives in the library's own device image: it
 * is not allocated by any call, and every GPU that loads the library's
 * device code holds it until the process exits.  Sizes with work to do
 * (M > 0, K > 0) whose workspace, qlinear_workspace_bytes(M, N, K,
 * hadamard_block), exceeds that capacity are then rejected with
 * QL_ERR_UNSUPPORTED before anything runs (for example M = 2048, N = 7168
 * fits; M = 12000, N = 7168 does not).
 *
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress, thread-safe); make that first call before
 * any stream capture.  With lazy module loading that lookup can be what
 * loads the library's device code, and with it the array, onto the device;
 * if it fails (e.g. the device is out of memory at that moment) the call
 * returns QL_ERR_CUDA and the next call looks it up again: only a lookup
 * that succeeded is kept.  All calls in the process share the
 * one array and it keeps whatever the last call left in it; nothing in it
 * needs to start at zero, because every byte this call reads was written
 * earlier in the same call.  Calls that may overlap on the GPU (different
 * streams, or different host threads on one device) race on the array:
 * order them, e.g. issue them on one stream.  The call allocates nothing. */
QL_API int qlinear_bwd_dx_noalloc(const void *dy, int dyt, int64_t M, int64_t N,
                                  const int8_t *wq, const float *sw, int64_t K,
                                  int hadamard_block, void *dx, int dxt,
                                  int32_t *d_status, void *stream);

/* Instrumentation (no effect on results).
 * ql_set_gemm_timing_events: the next n (<= 16) int8 GEMM kernels that the
 * calling host thread launches record the cudaEvent_t before[i] on their
 * stream right before the i-th launch and after[i] right after it, so a
 * caller can time the GEMMs alone inside layer calls (qlinear_bwd launches
 * two).  After n launches, or with n = 0, nothing is recorded.  The events
 * (host arrays of cudaEvent_t passed as void*) are the caller's; the library
 * copies the handles and only records them.
 * ql_kernel_launches: number of CUDA kernels this library has launched in the
 * process so far (all threads). */
QL_API void ql_set_gemm_timing_events(void *const *before, void *const *after, int n);
QL_API uint64_t ql_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
