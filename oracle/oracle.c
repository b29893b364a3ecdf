/*
 * CPU oracle for the INT8 quantized-training Linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * statement of what the layer computes.  Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the CUDA library never does,
 * and it shares no code, header, table or constant generator with it.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 *        (oracle/build.py).  All float arithmetic is IEEE binary32 with
 *        round-to-nearest-even and no contraction of a*b+c into an FMA,
 *        because float results here decide integer codes that must agree
 *        bit for bit with the GPU; the only float64 steps are the ones the
 *        text below names (host-side constants, the bias-gradient sum, the
 *        direction norm).
 *
 * Sources (web pages, cited by title and part):
 *   [QT]  mini_trainer "docs/quantized-training.md": intro paragraph (INT8
 *         weights and saved Linear inputs, integer forward/backward matrix
 *         products, no floating master weight; biases, gradients and
 *         optimizer state stay floating point); feature table rows
 *         "Row-wise weight normalization", "Inputs and inference",
 *         "Optimizers"; the paragraph after the table (updates requantize
 *         stochastically); the paragraph on contractions above 131,071.
 *   [CR]  OneTrainer PR #1681 "Int8 conv rot": opening summary (block-Hadamard
 *         rotation from a precomputed buffer), commit note item 1 (activations
 *         quantized per row on every call), item 2 ((xR)(WR)^T = xW^T, rotate
 *         x instead of un-rotating W), item 3 (orthogonality 5.96e-08, the
 *         torch._int_mm row floor), and the closing Summary.
 *   [PX]  Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
 *         1, 2, 3", SC'11 - the Philox4x32 counter-based generator.
 *
 * Readings where the pages leave a step open:
 *   - Per-row symmetric scale s = amax/127, codes rne(t * (127/amax)) clamped
 *     to [-127,127]; a zero row gets s = 0 and zero codes (flagged when the
 *     caller rejects zero rows, as [QT] rejects zero directions).
 *   - Block Hadamard = Sylvester order, butterflies h = 1,2,...,B/2, then one
 *     multiply by c = fl32(1/sqrt(B)).
 *   - dX of a rotated layer is rotated back with the same (symmetric) R.
 *   - Philox counter = (e>>2 lo, e>>2 hi, step lo, step hi), key = seed,
 *     word e&3, u24 = word >> 8, e = n*K + k.
 *   - AdamW in the decoupled textbook form with host constants rounded once.
 *   - Weight norm: direction v = s_v*q, effective row g*q/||q||; the direction
 *     gradient reduction order is pinned (see ref_update_sr).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status bits returned by the oracle.  They use the bit positions that the
 * C ABI uses for its device status word (1 << status code), declared here on
 * their own so the oracle needs nothing from the library. */
#define ORC_BIT_ARG        (1u << 1)
#define ORC_BIT_SHAPE      (1u << 2)
#define ORC_BIT_ZERO_ROW   (1u << 4)
#define ORC_BIT_NONFINITE  (1u << 5)
#define ORC_BIT_UNSUPP     (1u << 6)

#define ORC_REJECT_ZERO_ROWS 1u

/* Largest contraction whose int32 dot products cannot overflow for any int8
 * operands (|a|, |b| <= 128): floor((2^31 - 1) / 128^2) = 131,071 ([QT],
 * contraction paragraph). */
#define ORC_MAX_CONTRACTION 131071

/* ------------------------------------------------------------------ */
/* Block Hadamard rotation ([CR] summary; Summary para)                */
/* ------------------------------------------------------------------ */

/* c = 1/sqrt(B), computed in float64 and rounded once to float32. */
float ref_hadamard_scale(int B) { return (float)(1.0 / sqrt((double)B)); }

static int valid_block(int B) {
    if (B == 0) return 1;
    if (B < 2 || B > 256) return 0;
    return (B & (B - 1)) == 0;
}

/* One block of B values, in place: the Sylvester butterflies in order
 * h = 1, 2, 4, ..., B/2, each pair (v[j], v[j+h]) -> (v[j]+v[j+h], v[j]-v[j+h]),
 * then every value times c.  Equals v * H_B / sqrt(B) up to float rounding,
 * with H_B the Sylvester Hadamard matrix (symmetric, H_B H_B = B I). */
static void fwht_block(float *v, int B) {
    for (int h = 1; h < B; h <<= 1) {
        for (int i = 0; i < B; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = v[j];
                float b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
    float c = ref_hadamard_scale(B);
    for (int i = 0; i < B; ++i) v[i] = v[i] * c;
}

/* y[r, :] = x[r, :] R for every row, R = blockdiag(H_B/sqrt(B)).  x and y may
 * alias.  Returns 0 or ORC_BIT_SHAPE (bad block or cols % B != 0). */
uint32_t ref_hadamard_rows(const float *x, int64_t ldx, float *y, int64_t ldy,
                           int64_t rows, int64_t cols, int B) {
    if (!valid_block(B) || B == 0 || cols % B != 0) return ORC_BIT_SHAPE;
    float *t = (float *)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(float));
    for (int64_t r = 0; r < rows; ++r) {
        memcpy(t, x + r * ldx, (size_t)cols * sizeof(float));
        for (int64_t b0 = 0; b0 < cols; b0 += B) fwht_block(t + b0, B);
        memcpy(y + r * ldy, t, (size_t)cols * sizeof(float));
    }
    free(t);
    return 0;
}

/* The dense form, for checks only: R as a [B,B] row-major float64 matrix. */
void ref_hadamard_matrix_f64(int B, double *R) {
    double c = 1.0 / sqrt((double)B);
    for (int i = 0; i < B; ++i)
        for (int j = 0; j < B; ++j) {
            /* Sylvester: H[i][j] = (-1)^popcount(i & j) */
            int p = __builtin_popcount((unsigned)(i & j)) & 1;
            R[(int64_t)i * B + j] = p ? -c : c;
        }
}

/* ------------------------------------------------------------------ */
/* Per-row symmetric INT8 quantization ([CR] item 1; [QT] intro)       */
/* ------------------------------------------------------------------ */

/* For each row r: t = x[r,:] (* col_scale, if given) (-> t R, if B > 0);
 * amax = max |t|; s[r] = amax/127; q[r,:] = clamp(rne(t * (127/amax)), +-127).
 * amax == 0: s = 0, codes 0, and ORC_BIT_ZERO_ROW when flags rejects zero
 * rows.  A non-finite t sets ORC_BIT_NONFINITE (codes then unspecified). */
uint32_t ref_quantize_rows(const float *x, int64_t rows, int64_t cols, int64_t ldx,
                           const float *col_scale, int B, uint32_t flags,
                           int8_t *q, int64_t ldq, float *s) {
    if (!valid_block(B)) return ORC_BIT_ARG;
    if (B > 0 && cols % B != 0) return ORC_BIT_SHAPE;
    uint32_t st = 0;
    float *t = (float *)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(float));
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * ldx;
        for (int64_t k = 0; k < cols; ++k)
            t[k] = col_scale ? xr[k] * col_scale[k] : xr[k];
        if (B > 0)
            for (int64_t b0 = 0; b0 < cols; b0 += B) fwht_block(t + b0, B);
        float amax = 0.0f;
        int bad = 0;
        for (int64_t k = 0; k < cols; ++k) {
            if (!isfinite(t[k])) bad = 1;
            float a = fabsf(t[k]);
            if (a > amax) amax = a;
        }
        if (bad) st |= ORC_BIT_NONFINITE;
        int8_t *qr = q + r * ldq;
        if (amax == 0.0f) {
            s[r] = 0.0f;
            for (int64_t k = 0; k < cols; ++k) qr[k] = 0;
            if (flags & ORC_REJECT_ZERO_ROWS) st |= ORC_BIT_ZERO_ROW;
            continue;
        }
        float inv = 127.0f / amax;
        s[r] = amax / 127.0f;
        for (int64_t k = 0; k < cols; ++k) {
            float v = t[k] * inv;
            float rq = nearbyintf(v); /* default rounding mode: to nearest even */
            if (rq > 127.0f) rq = 127.0f;
            if (rq < -127.0f) rq = -127.0f;
            qr[k] = (int8_t)rq;
        }
    }
    free(t);
    return st;
}

/* ------------------------------------------------------------------ */
/* Dequantization back to the original basis ([CR] third commit note,  */
/* item 2: unquantized_weight un-rotates for LoRA and offload callers)  */
/* ------------------------------------------------------------------ */

/* w[n,k] = s[n] * (float)q[n,k] (one float32 product), then for B > 0 each
 * row times R, which is its own inverse (H_B H_B = B I), so a weight that
 * was rotated before quantization comes back in its original basis. */
uint32_t ref_dequantize(const int8_t *q, int64_t ldq, const float *s, int64_t N, int64_t K,
                        int B, float *w, int64_t ldw) {
    if (!valid_block(B)) return ORC_BIT_ARG;
    if (B > 0 && K % B != 0) return ORC_BIT_SHAPE;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) w[n * ldw + k] = (float)q[n * ldq + k] * s[n];
    if (B > 0) return ref_hadamard_rows(w, ldw, w, ldw, N, K, B);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Integer GEMMs ([CR] summary: int8 x int8 -> int32 as torch._int_mm; */
/* [QT] intro: integer forward and backward matrix products)           */
/* ------------------------------------------------------------------ */

static int fits_i32(int64_t v) { return v >= INT32_MIN && v <= INT32_MAX; }

/* out[m,n] = sum_c A[m,c] * B[n,c]   (both operands contraction-contiguous).
 * Exact int64 sums; ORC_BIT_UNSUPP if a sum leaves the int32 range. */
uint32_t ref_gemm_nt(const int8_t *A, int64_t lda, const int8_t *Bm, int64_t ldb,
                     int64_t M, int64_t N, int64_t C, int32_t *out, int64_t ldo) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            const int8_t *a = A + m * lda, *b = Bm + n * ldb;
            for (int64_t c = 0; c < C; ++c) acc += (int64_t)a[c] * (int64_t)b[c];
            if (!fits_i32(acc)) return ORC_BIT_UNSUPP;
            out[m * ldo + n] = (int32_t)acc;
        }
    return 0;
}

/* out[m,n] = sum_c A[m,c] * B[c,n]   (B stored contraction-major).
 * The exact integer sum of each output is accumulated row by row. */
uint32_t ref_gemm_nn(const int8_t *A, int64_t lda, const int8_t *Bm, int64_t ldb,
                     int64_t M, int64_t N, int64_t C, int32_t *out, int64_t ldo) {
    int64_t *acc = (int64_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(int64_t));
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) acc[n] = 0;
        for (int64_t c = 0; c < C; ++c) {
            int64_t a = A[m * lda + c];
            if (a == 0) continue;
            const int8_t *b = Bm + c * ldb;
            for (int64_t n = 0; n < N; ++n) acc[n] += a * (int64_t)b[n];
        }
        for (int64_t n = 0; n < N; ++n) {
            if (!fits_i32(acc[n])) { free(acc); return ORC_BIT_UNSUPP; }
            out[m * ldo + n] = (int32_t)acc[n];
        }
    }
    free(acc);
    return 0;
}

/* out[m,n] = sum_c A[c,m] * B[c,n]   (both stored contraction-major). */
uint32_t ref_gemm_tn(const int8_t *A, int64_t lda, const int8_t *Bm, int64_t ldb,
                     int64_t M, int64_t N, int64_t C, int32_t *out, int64_t ldo) {
    int64_t *acc = (int64_t *)calloc((size_t)(M * N > 0 ? M * N : 1), sizeof(int64_t));
    for (int64_t c = 0; c < C; ++c) {
        const int8_t *a = A + c * lda, *b = Bm + c * ldb;
        for (int64_t m = 0; m < M; ++m) {
            int64_t am = a[m];
            if (am == 0) continue;
            int64_t *row = acc + m * N;
            for (int64_t n = 0; n < N; ++n) row[n] += am * (int64_t)b[n];
        }
    }
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            if (!fits_i32(acc[m * N + n])) { free(acc); return ORC_BIT_UNSUPP; }
            out[m * ldo + n] = (int32_t)acc[m * N + n];
        }
    free(acc);
    return 0;
}

/* The same two products with int64 outputs and no range limit: contractions
 * longer than 131,071 combine their bounded int32 partial dot products in
 * int64 before scaling ([QT], contraction paragraph).  Integer addition is
 * associative, so any chunking of the contraction gives this exact sum. */
void ref_gemm_nn64(const int8_t *A, int64_t lda, const int8_t *Bm, int64_t ldb,
                   int64_t M, int64_t N, int64_t C, int64_t *out, int64_t ldo) {
    for (int64_t m = 0; m < M; ++m) {
        int64_t *acc = out + m * ldo;
        for (int64_t n = 0; n < N; ++n) acc[n] = 0;
        for (int64_t c = 0; c < C; ++c) {
            int64_t a = A[m * lda + c];
            if (a == 0) continue;
            const int8_t *b = Bm + c * ldb;
            for (int64_t n = 0; n < N; ++n) acc[n] += a * (int64_t)b[n];
        }
    }
}

void ref_gemm_tn64(const int8_t *A, int64_t lda, const int8_t *Bm, int64_t ldb,
                   int64_t M, int64_t N, int64_t C, int64_t *out, int64_t ldo) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) out[m * ldo + n] = 0;
    for (int64_t c = 0; c < C; ++c) {
        const int8_t *a = A + c * lda, *b = Bm + c * ldb;
        for (int64_t m = 0; m < M; ++m) {
            int64_t am = a[m];
            if (am == 0) continue;
            int64_t *row = out + m * ldo;
            for (int64_t n = 0; n < N; ++n) row[n] += am * (int64_t)b[n];
        }
    }
}

/* ------------------------------------------------------------------ */
/* Layer forward ([CR] item 1 and Summary; [QT] intro and table row     */
/* "Inputs and inference": bias, batched and single-sample inputs)      */
/* ------------------------------------------------------------------ */

/* x [M,K] float; W_q [N,K] int8 with per-row scale s_w (already in the
 * rotated basis when B > 0).  Saves X_q [M,K] and s_x [M] for backward and
 * writes y[m,n] = ((float)acc[m,n] * s_x[m]) * s_w[n] + bias[n] in float32. */
uint32_t ref_fwd(const float *x, int64_t M, int64_t K, const int8_t *wq, const float *sw,
                 int64_t N, const float *bias, int B, float *y, int8_t *xq, float *sx) {
    if (K > ORC_MAX_CONTRACTION) return ORC_BIT_UNSUPP;
    uint32_t st = ref_quantize_rows(x, M, K, K, NULL, B, 0u, xq, K, sx);
    if (st & (ORC_BIT_ARG | ORC_BIT_SHAPE)) return st;
    int32_t *acc = (int32_t *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(int32_t));
    st |= ref_gemm_nt(xq, K, wq, K, M, N, K, acc, N);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float v = ((float)acc[m * N + n] * sx[m]) * sw[n];
            y[m * N + n] = bias ? v + bias[n] : v;
        }
    free(acc);
    return st;
}

/* The same forward from an input that is already quantized (codes xq [M,K]
 * and row scales sx [M] in the layer's format, e.g. the SwiGLU gate's
 * quantized h): y[m,n] = ((float)acc[m,n] * sx[m]) * s_w[n] + bias[n]. */
uint32_t ref_fwd_quantized(const int8_t *xq, const float *sx, int64_t M, int64_t K,
                           const int8_t *wq, const float *sw, int64_t N, const float *bias,
                           float *y) {
    if (K > ORC_MAX_CONTRACTION) return ORC_BIT_UNSUPP;
    int32_t *acc = (int32_t *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(int32_t));
    uint32_t st = ref_gemm_nt(xq, K, wq, K, M, N, K, acc, N);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float v = ((float)acc[m * N + n] * sx[m]) * sw[n];
            y[m * N + n] = bias ? v + bias[n] : v;
        }
    free(acc);
    return st;
}

/* ------------------------------------------------------------------ */
/* The forward's bf16 route ([CR] third commit note, items 1 and 2: the  */
/* activations are rotated instead of the weight being un-rotated, and   */
/* they are not quantized)                                              */
/* ------------------------------------------------------------------ */

/* float32 -> bf16 (the upper 16 bits of a float32), rounding to nearest with
 * ties to even; a NaN stays a (quiet) NaN.  Returned as the float32 it
 * represents. */
float ref_round_bf16(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) {
        u = (u | 0x00400000u) & 0xFFFF0000u;
    } else {
        uint32_t lsb = (u >> 16) & 1u;
        u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/* xr = bf16(x R) (x itself, rounded, when B = 0); the weight enters as its
 * codes q, exact in bf16; y[m,n] = ((float)(sum_k xr[m,k] q[n,k])) * s_w[n]
 * + bias[n], with every product exact and the sum taken in float64.  The
 * tensor cores accumulate in float32 in an order of their own, so a kernel
 * matches this within a rounding bound, not bit for bit.  xr [M,K] is
 * returned for the checks. */
uint32_t ref_fwd_bf16(const float *x, int64_t M, int64_t K, const int8_t *wq, const float *sw,
                      int64_t N, const float *bias, int B, float *y, float *xr) {
    if (!valid_block(B)) return ORC_BIT_ARG;
    if (B > 0 && K % B != 0) return ORC_BIT_SHAPE;
    uint32_t st = 0;
    if (B > 0) st = ref_hadamard_rows(x, K, xr, K, M, K, B);
    else memcpy(xr, x, (size_t)(M * K) * sizeof(float));
    for (int64_t i = 0; i < M * K; ++i) xr[i] = ref_round_bf16(xr[i]);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            const float *a = xr + m * K;
            const int8_t *b = wq + n * K;
            for (int64_t k = 0; k < K; ++k) acc += (double)a[k] * (double)b[k];
            float v = (float)acc * sw[n];
            y[m * N + n] = bias ? v + bias[n] : v;
        }
    return st;
}

/* ------------------------------------------------------------------ */
/* Backward preparation (the layer's formulas for dX and dW)           */
/* ------------------------------------------------------------------ */

/* Row part: t'[m,n] = dY[m,n] * s_w[n], quantized per row -> dYq_r, s1[m]. */
uint32_t ref_bwd_prep_rows(const float *dy, int64_t M, int64_t N, const float *sw,
                           int8_t *dyq_r, float *s1) {
    return ref_quantize_rows(dy, M, N, N, sw, 0, 0u, dyq_r, N, s1);
}

/* Column part: t''[m,n] = dY[m,n] * s_x[m]; per column n: amax over m,
 * s2[n] = amax/127, dYq_c[m,n] = clamp(rne(t'' * (127/amax)), +-127), stored
 * [M,N] like dY; a zero column gets s2 = 0 and zero codes.  db[n] (if given)
 * = sum over m of dY[m,n], summed in float64 and rounded once. */
uint32_t ref_bwd_prep_cols(const float *dy, int64_t M, int64_t N, const float *sx,
                           int8_t *dyq_c, float *s2, float *db) {
    uint32_t st = 0;
    for (int64_t n = 0; n < N; ++n) {
        float amax = 0.0f;
        double sum = 0.0;
        int bad = 0;
        for (int64_t m = 0; m < M; ++m) {
            float t = dy[m * N + n] * sx[m];
            if (!isfinite(t)) bad = 1;
            float a = fabsf(t);
            if (a > amax) amax = a;
            sum += (double)dy[m * N + n];
        }
        if (bad) st |= ORC_BIT_NONFINITE;
        if (db) db[n] = (float)sum;
        if (amax == 0.0f) {
            s2[n] = 0.0f;
            for (int64_t m = 0; m < M; ++m) dyq_c[m * N + n] = 0;
            continue;
        }
        float inv = 127.0f / amax;
        s2[n] = amax / 127.0f;
        for (int64_t m = 0; m < M; ++m) {
            float t = dy[m * N + n] * sx[m];
            float rq = nearbyintf(t * inv);
            if (rq > 127.0f) rq = 127.0f;
            if (rq < -127.0f) rq = -127.0f;
            dyq_c[m * N + n] = (int8_t)rq;
        }
    }
    return st;
}

/* dX[m,k] = (float)(sum_n dYq_r[m,n] W_q[n,k]) * s1[m]; then, for a rotated
 * layer (B > 0), each row of dX times R (R symmetric, so this is dX' R^T).
 * The sum is exact in int64 for any N: above 131,071 output classes it is
 * the int64 combination of int32 chunk sums ([QT], contraction paragraph),
 * converted to float32 once (round to nearest even). */
uint32_t ref_bwd_dx(const float *dy, int64_t M, int64_t N, const int8_t *wq,
                    const float *sw, int64_t K, int B, float *dx,
                    int8_t *dyq_r, float *s1) {
    if (!valid_block(B)) return ORC_BIT_ARG;
    if (B > 0 && K % B != 0) return ORC_BIT_SHAPE;
    uint32_t st = ref_bwd_prep_rows(dy, M, N, sw, dyq_r, s1);
    int64_t *acc = (int64_t *)malloc((size_t)(M * K > 0 ? M * K : 1) * sizeof(int64_t));
    ref_gemm_nn64(dyq_r, N, wq, K, M, K, N, acc, K);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) dx[m * K + k] = (float)acc[m * K + k] * s1[m];
    free(acc);
    if (B > 0) st |= ref_hadamard_rows(dx, K, dx, K, M, K, B);
    return st;
}

/* dW[n,k] = (float)(sum_m dYq_c[m,n] X_q[m,k]) * s2[n]; db as above.  The
 * sum over tokens is exact in int64 for any M (int64 combination of int32
 * chunk sums above 131,071 tokens). */
uint32_t ref_bwd_dw(const float *dy, int64_t M, int64_t N, const int8_t *xq,
                    const float *sx, int64_t K, float *dw, float *db,
                    int8_t *dyq_c, float *s2) {
    uint32_t st = ref_bwd_prep_cols(dy, M, N, sx, dyq_c, s2, db);
    int64_t *acc = (int64_t *)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(int64_t));
    ref_gemm_tn64(dyq_c, N, xq, K, N, K, M, acc, K);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) dw[n * K + k] = (float)acc[n * K + k] * s2[n];
    free(acc);
    return st;
}

/* ------------------------------------------------------------------ */
/* Philox4x32-10 ([PX], section 4: the Philox S-box and key schedule)   */
/* ------------------------------------------------------------------ */

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u /* golden ratio */
#define PHILOX_W1 0xBB67AE85u /* sqrt(3) - 1 */

static void mulhilo32(uint32_t a, uint32_t b, uint32_t *hi, uint32_t *lo) {
    uint64_t p = (uint64_t)a * (uint64_t)b;
    *hi = (uint32_t)(p >> 32);
    *lo = (uint32_t)p;
}

/* Ten rounds; round i uses key (k0 + i*W0, k1 + i*W1) mod 2^32. */
void ref_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint32_t hi0, lo0, hi1, lo1;
        mulhilo32(PHILOX_M0, c0, &hi0, &lo0);
        mulhilo32(PHILOX_M1, c2, &hi1, &lo1);
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 24-bit uniform that decides the stochastic rounding of element e
 * (e = n*K + k, the logical index) at optimizer step `step`. */
uint32_t ref_sr_u24(uint64_t seed, uint64_t step, uint64_t e) {
    uint64_t blk = e >> 2;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)step,
                       (uint32_t)(step >> 32)};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    ref_philox4x32_10(ctr, key, out);
    return out[e & 3] >> 8;
}

/* ------------------------------------------------------------------ */
/* Stochastic requantization update ([QT] paragraph after the feature    */
/* table; table rows "Optimizers", "Row-wise weight normalization")     */
/* ------------------------------------------------------------------ */

/* Stochastic rounding of value v (|v| <= 127 up to rounding) with uniform
 * u24: floor(v) + 1 with probability frac(v), decided as u24 < frac * 2^24. */
static float sr_round(float v, uint32_t u24) {
    float f = floorf(v);
    float frac = v - f; /* exact */
    float r = ((float)u24 < frac * 16777216.0f) ? f + 1.0f : f;
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return r;
}

/* Host-side AdamW constants, each computed in float64 and rounded once. */
typedef struct {
    float a;     /* 1 - lr*wd             (decoupled weight decay factor) */
    float st;    /* lr / (1 - b1^t)       (bias-corrected step size)      */
    float rbc2;  /* 1 / sqrt(1 - b2^t)    (second-moment bias correction, on the root) */
    float b1, b2, omb1, omb2, eps, lr;
} adamw_consts;

static adamw_consts adamw_setup(float lr, float b1, float b2, float eps, float wd,
                                uint64_t step) {
    adamw_consts c;
    double t = (double)step;
    c.a = (float)(1.0 - (double)lr * (double)wd);
    c.st = (float)((double)lr / (1.0 - pow((double)b1, t)));
    c.rbc2 = (float)(1.0 / sqrt(1.0 - pow((double)b2, t)));
    c.b1 = b1;
    c.b2 = b2;
    c.omb1 = (float)(1.0 - (double)b1);
    c.omb2 = (float)(1.0 - (double)b2);
    c.eps = eps;
    c.lr = lr;
    return c;
}

/* One AdamW step of one element (decoupled weight decay, Loshchilov & Hutter):
 * w1 = w*a; m' = b1*m + (1-b1)*g; v' = b2*v + (1-b2)*(g*g);
 * w' = w1 - st * (m' / (sqrt(v') * rbc2 + eps)),
 * i.e. sqrt(v'/(1-b2^t)) taken as sqrt(v') / sqrt(1-b2^t) with the
 * reciprocal root rounded once on the host. */
static float adamw_elem(const adamw_consts *c, float w, float g, float *m, float *v) {
    float w1 = w * c->a;
    float mn = c->b1 * (*m) + c->omb1 * g;
    float vn = c->b2 * (*v) + c->omb2 * (g * g);
    float den = sqrtf(vn) * c->rbc2 + c->eps;
    *m = mn;
    *v = vn;
    return w1 - c->st * (mn / den);
}

/* Requantize one row of updated float values w[0..K) stochastically: new
 * per-row scale from amax, codes by sr_round with the element's u24. */
static uint32_t sr_requant_row(const float *w, int64_t K, int64_t n, uint64_t seed,
                               uint64_t step, int8_t *q, float *s) {
    float amax = 0.0f;
    uint32_t st = 0;
    for (int64_t k = 0; k < K; ++k) {
        if (!isfinite(w[k])) st |= ORC_BIT_NONFINITE;
        float a = fabsf(w[k]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 0.0f;
        for (int64_t k = 0; k < K; ++k) q[k] = 0;
        return st;
    }
    float inv = 127.0f / amax;
    *s = amax / 127.0f;
    for (int64_t k = 0; k < K; ++k) {
        uint32_t u = ref_sr_u24(seed, step, (uint64_t)n * (uint64_t)K + (uint64_t)k);
        q[k] = (int8_t)sr_round(w[k] * inv, u);
    }
    return st;
}

/* Virtual-lane count of the pinned direction-gradient reduction. */
#define WN_LANES 256
#define WN_GROUP 16

/* sum_k a[k]*b[k] in the pinned order: the K elements are cut into groups of
 * 16 consecutive elements; group j belongs to virtual lane j mod 256; each
 * lane adds its products in increasing k starting from +0; then the 256 lane
 * partials are combined by an xor butterfly with offsets 128, 64, ..., 1
 * (partial[l] + partial[l ^ off]; every lane ends with the same value). */
static float pinned_dot(const float *a, const int8_t *qb, float nq, int64_t K, float *qhat) {
    float p[WN_LANES];
    for (int l = 0; l < WN_LANES; ++l) p[l] = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        int l = (int)((k / WN_GROUP) % WN_LANES);
        float qh = (float)qb[k] / nq;
        qhat[k] = qh;
        p[l] = p[l] + a[k] * qh;
    }
    for (int off = WN_LANES / 2; off >= 1; off >>= 1)
        for (int l = 0; l < off; ++l) p[l] = p[l] + p[l + off];
    return p[0];
}

/* The float optimizer step of one row n (no requantization).
 *   kind 0 = SGD:   w' = w - lr*g            (no momentum; wd must be 0)
 *   kind 1 = AdamW: as adamw_elem, moments m, v float32 updated in place.
 * Plain weights: w[k] = s[n]*q[n,k]; grad = dL/dw.
 * Row-wise weight norm (g != NULL): the stored int8 row is the direction
 * v = s[n]*q[n,:]; the effective row is g[n]*q/||q|| with ||q|| =
 * fl32(sqrt(sum q^2)) (exact integer sum); grad = dL/d(effective row):
 *   qhat = q/||q||, dg = pinned_dot(grad, qhat),
 *   dv = (g[n] / (s[n]*||q||)) * (grad - dg*qhat).
 * The optimizer steps v with dv (moments m, v) and g[n] with dg (moments
 * g_m[n], g_v[n]).  A zero initial direction returns ORC_BIT_ZERO_ROW and
 * changes nothing.  The updated float row is left in w[0..K). */
static uint32_t row_step(const int8_t *qr, float sn, const float *gr, int64_t K, int64_t n,
                         int kind, const adamw_consts *c, float *mr, float *vr,
                         float *g, float *g_m, float *g_v, float *w, float *qhat) {
    if (g) {
        int64_t ss = 0;
        for (int64_t k = 0; k < K; ++k) ss += (int64_t)qr[k] * (int64_t)qr[k];
        if (ss == 0) return ORC_BIT_ZERO_ROW;
        float nq = (float)sqrt((double)ss);
        float dg = pinned_dot(gr, qr, nq, K, qhat);
        float coef = g[n] / (sn * nq);
        for (int64_t k = 0; k < K; ++k) {
            float dv = coef * (gr[k] - dg * qhat[k]);
            float wv = sn * (float)qr[k];
            w[k] = (kind == 1) ? adamw_elem(c, wv, dv, &mr[k], &vr[k]) : wv - c->lr * dv;
        }
        g[n] = (kind == 1) ? adamw_elem(c, g[n], dg, &g_m[n], &g_v[n]) : g[n] - c->lr * dg;
    } else {
        for (int64_t k = 0; k < K; ++k) {
            float wv = sn * (float)qr[k];
            w[k] = (kind == 1) ? adamw_elem(c, wv, gr[k], &mr[k], &vr[k]) : wv - c->lr * gr[k];
        }
    }
    return 0;
}

static uint32_t check_update_args(int kind, float wd, uint64_t step) {
    if (step < 1 || (kind != 0 && kind != 1)) return ORC_BIT_ARG;
    if (kind == 0 && wd != 0.0f) return ORC_BIT_ARG;
    return 0;
}

/* The float step of every row, written to w_out [N,K] (rows with a zero
 * direction keep s*q); moments and g updated in place.  For checks of the
 * optimizer arithmetic on its own. */
uint32_t ref_update_float(const int8_t *q, const float *s, const float *grad, int64_t N, int64_t K,
                          int kind, float lr, float b1, float b2, float eps, float wd,
                          float *m, float *v, uint64_t step,
                          float *g, float *g_m, float *g_v, float *w_out) {
    uint32_t st = check_update_args(kind, wd, step);
    if (st) return st;
    adamw_consts c = adamw_setup(lr, b1, b2, eps, wd, step);
    float *qhat = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
        float *w = w_out + n * K;
        uint32_t r = row_step(q + n * K, s[n], grad + n * K, K, n, kind, &c,
                              m ? m + n * K : NULL, v ? v + n * K : NULL,
                              g, g_m, g_v, w, qhat);
        if (r) {
            for (int64_t k = 0; k < K; ++k) w[k] = s[n] * (float)q[n * K + k];
            st |= r;
        }
    }
    free(qhat);
    return st;
}

/* One optimizer step with stochastic requantization of an int8 [N,K] weight,
 * in place: row_step, then sr_requant_row of the updated row (seed, step).
 * Rows with a zero initial direction are left untouched.  step >= 1.
 * The arrays hold rows n0 .. n0+N-1 of the weight: the row index that keys
 * the random stream is n0 + n (so a slice of rows can be checked alone). */
uint32_t ref_update_sr(int8_t *q, float *s, const float *grad, int64_t N, int64_t K,
                       int kind, float lr, float b1, float b2, float eps, float wd,
                       float *m, float *v, uint64_t seed, uint64_t step,
                       float *g, float *g_m, float *g_v, int64_t n0) {
    uint32_t st = check_update_args(kind, wd, step);
    if (st) return st;
    adamw_consts c = adamw_setup(lr, b1, b2, eps, wd, step);
    float *w = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    float *qhat = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
        uint32_t r = row_step(q + n * K, s[n], grad + n * K, K, n, kind, &c,
                              m ? m + n * K : NULL, v ? v + n * K : NULL,
                              g, g_m, g_v, w, qhat);
        if (r) { st |= r; continue; }
        st |= sr_requant_row(w, K, n0 + n, seed, step, q + n * K, &s[n]);
    }
    free(w);
    free(qhat);
    return st;
}

/* Expected value of the stochastically rounded code of v over all 2^24
 * uniforms, by enumeration (used by the unbiasedness checks). */
double ref_sr_expectation_enum(float v) {
    double total = 0.0;
    for (uint32_t u = 0; u < (1u << 24); ++u) total += (double)sr_round(v, u);
    return total / 16777216.0;
}

/* ------------------------------------------------------------------ */
/* SwiGLU gate of the three-projection MLP (the MLP training step the   */
/* layer is measured in: w1 and w3 take the same input, w2 takes h):    */
/* h = silu(a) * b with silu(a) = a / (1 + e^-a)                        */
/* ------------------------------------------------------------------ */

/* e^x in float32, the same float32 steps wherever it is evaluated, so a
 * code that depends on it is reproducible bit for bit (library expf
 * implementations differ in the last place).  Method: Cody and Waite's
 * argument reduction (W. J. Cody, W. Waite, "Software Manual for the
 * Elementary Functions", 1980): n = rint(x * log2(e)), r = x - n*ln2 with
 * ln2 split into its float32 value C1 and the remainder C2, each step one
 * correctly rounded fused multiply-add; then e^r from its Taylor series
 * sum_{k=0..7} r^k / k! by Horner's rule (|r| <= ln2/2 + tiny, so the first
 * omitted term r^8/8! is below 5.4e-9 relative); then times 2^n as two exact
 * powers of two (2^n1 * 2^n2, n1 = n/2), so the only rounding in the
 * subnormal range is the last product.  x is clamped to [-104, 89] first:
 * e^89 overflows float32 and e^-104 is below half the smallest subnormal. */
float ref_exp(float x) {
    if (x != x) return x;
    const float L2E = 1.44269504088896341f;            /* log2(e) */
    const float C1 = 0.693147182464599609375f;         /* fl32(ln 2) */
    const float C2 = -1.904654299957768e-09f;          /* ln 2 - C1 */
    static const float c[8] = {1.0f, 1.0f, 0.5f, 0.16666666666666666f,
                               0.041666666666666664f, 0.008333333333333333f,
                               0.001388888888888889f, 0.0001984126984126984f}; /* 1/k! */
    float xc = x > 89.0f ? 89.0f : (x < -104.0f ? -104.0f : x);
    float nf = rintf(xc * L2E);
    int n = (int)nf;
    float r = fmaf(-nf, C1, xc);
    r = fmaf(-nf, C2, r);
    float p = c[7];
    for (int k = 6; k >= 0; --k) p = fmaf(p, r, c[k]);
    int n1 = n / 2, n2 = n - n1;
    uint32_t b1 = (uint32_t)(n1 + 127) << 23, b2 = (uint32_t)(n2 + 127) << 23;
    float f1, f2;
    memcpy(&f1, &b1, 4);
    memcpy(&f2, &b2, 4);
    return (p * f1) * f2;
}

/* silu(a) = a / (1 + e^-a): one float32 addition and one IEEE division. */
static float ref_silu(float a) { return a / (1.0f + ref_exp(-a)); }

/* h[m, f] = silu(a[m, f]) * b[m, f] for the stacked pre-activations
 * ab [M, 2F] (a = columns 0..F-1, b = columns F..2F-1, pitch ldab). */
void ref_swiglu_h(const float *ab, int64_t M, int64_t F, int64_t ldab, float *h) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t f = 0; f < F; ++f) {
            const float a = ab[m * ldab + f], b = ab[m * ldab + F + f];
            h[m * F + f] = ref_silu(a) * b;
        }
}

/* The input of the MLP's second projection as that layer saves it: h per
 * row quantized exactly as the layer's forward quantizes its input (no
 * rotation): s_h[m] = amax/127, hq = clamp(rne(h * (127/amax)), +-127); a
 * zero row of h gives s_h = 0 and zero codes; a non-finite h sets
 * ORC_BIT_NONFINITE. */
uint32_t ref_swiglu_quantize(const float *ab, int64_t M, int64_t F, int64_t ldab,
                             int8_t *hq, float *sh) {
    float *h = (float *)malloc((size_t)(M * F > 0 ? M * F : 1) * sizeof(float));
    ref_swiglu_h(ab, M, F, ldab, h);
    uint32_t st = ref_quantize_rows(h, M, F, F, NULL, 0, 0u, hq, F, sh);
    free(h);
    return st;
}

/* The gate's backward: given dh [M, F] (the input gradient of the second
 * projection) and ab, the gradient at the stacked pre-activations
 * dab [M, 2F]:  with e = e^-a, d = 1 + e, sigma = 1/d, silu = a/d,
 *   da = (dh * b) * (sigma * (1 + a * (1 - sigma)))    (d silu/da)
 *   db = dh * silu
 * each operation one float32 rounding in the order written. */
void ref_swiglu_bwd(const float *ab, int64_t M, int64_t F, int64_t ldab, const float *dh,
                    float *dab) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t f = 0; f < F; ++f) {
            const float a = ab[m * ldab + f], b = ab[m * ldab + F + f];
            const float g = dh[m * F + f];
            const float d = 1.0f + ref_exp(-a);
            const float sigma = 1.0f / d;
            const float silu = a / d;
            const float ds = sigma * (1.0f + a * (1.0f - sigma));
            dab[m * 2 * F + f] = (g * b) * ds;
            dab[m * 2 * F + F + f] = g * silu;
        }
}

/* ------------------------------------------------------------------ */
/* MuonAuxAdamW ([QT] feature table, row "Optimizers": the third update  */
/* path it names).  The pages give only the name; the definition        */
/* followed is the published Muon optimizer (K. Jordan, Y. Jin, V. Boza,  */
/* J. You, F. Cesista, L. Newhouse, J. Bernstein, "Muon: An optimizer for */
/* hidden layers in neural networks", 2024) for the 2-D weights, with     */
/* AdamW for the float parameters (biases, magnitudes):                   */
/*   M' = beta*M + (1-beta)*G,  U = (1-beta)*G + beta*M'   (Nesterov)     */
/*   O = NS5(U): quintic Newton-Schulz on U/||U||_F, 5 steps              */
/*   w' = w*(1 - lr*wd) - lr*max(1, N/K)^0.5 * O, then the layer's         */
/*   stochastic requantization of each row.                               */
/* ------------------------------------------------------------------ */

/* Momentum and Nesterov blend, float32, one rounding per operation in the
 * order written; omb = fl32(1 - beta) computed in float64.  M is updated in
 * place; U receives the blended update. */
void ref_muon_momentum(const float *G, float *M, int64_t n, float beta, float *U) {
    const float omb = (float)(1.0 - (double)beta);
    for (int64_t i = 0; i < n; ++i) {
        const float m = beta * M[i] + omb * G[i];
        M[i] = m;
        U[i] = omb * G[i] + beta * m;
    }
}

/* O = NS5(U) in float64.  X = U, or U^T when U has more rows than columns
 * (so X is r x c with r <= c); X = X / (||X||_F + 1e-7); then `steps` times
 *   A = X X^T;  B = b*A + c*(A A);  X = a*X + B X
 * with (a, b, c) = (3.4445, -4.7750, 2.0315); O = X (transposed back).
 * Acting on the singular values alone, each step maps s -> a s + b s^3 +
 * c s^5, so O = U_svd p(S/(||U||_F + 1e-7)) V_svd^T with p the step applied
 * `steps` times.  U [R, C] float row-major, O [R, C] double row-major. */
void ref_newton_schulz5(const float *U, int64_t R, int64_t C, int steps, double *O) {
    const double a = 3.4445, b = -4.7750, c = 2.0315;
    const int tr = R > C;
    const int64_t r = tr ? C : R, cc = tr ? R : C;
    double *X = (double *)malloc((size_t)(r * cc > 0 ? r * cc : 1) * sizeof(double));
    double *Y = (double *)malloc((size_t)(r * cc > 0 ? r * cc : 1) * sizeof(double));
    double *A = (double *)malloc((size_t)(r * r > 0 ? r * r : 1) * sizeof(double));
    double *B = (double *)malloc((size_t)(r * r > 0 ? r * r : 1) * sizeof(double));
    double nrm = 0.0;
    for (int64_t i = 0; i < r; ++i)
        for (int64_t j = 0; j < cc; ++j) {
            const double v = tr ? (double)U[j * C + i] : (double)U[i * C + j];
            X[i * cc + j] = v;
            nrm += v * v;
        }
    nrm = sqrt(nrm) + 1e-7;
    for (int64_t i = 0; i < r * cc; ++i) X[i] /= nrm;
    for (int s = 0; s < steps; ++s) {
        for (int64_t i = 0; i < r; ++i)           /* A = X X^T */
            for (int64_t j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < cc; ++k) acc += X[i * cc + k] * X[j * cc + k];
                A[i * r + j] = acc;
            }
        for (int64_t i = 0; i < r; ++i)           /* B = b A + c A A */
            for (int64_t j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < r; ++k) acc += A[i * r + k] * A[k * r + j];
                B[i * r + j] = b * A[i * r + j] + c * acc;
            }
        for (int64_t i = 0; i < r; ++i)           /* X = a X + B X */
            for (int64_t j = 0; j < cc; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < r; ++k) acc += B[i * r + k] * X[k * cc + j];
                Y[i * cc + j] = a * X[i * cc + j] + acc;
            }
        double *t = X;
        X = Y;
        Y = t;
    }
    for (int64_t i = 0; i < r; ++i)
        for (int64_t j = 0; j < cc; ++j) {
            if (tr) O[j * C + i] = X[i * cc + j];
            else O[i * C + j] = X[i * cc + j];
        }
    free(X);
    free(Y);
    free(A);
    free(B);
}

/* One Muon step of an int8 weight [N, K] with stochastic requantization, in
 * place, from the orthogonalized update O (float32 [N, K]):
 *   w = s*q;  w' = w*a - st*O,  a = fl32(1 - lr*wd), st = fl32(lr*max(1, N/K)^0.5)
 * (constants in float64, rounded once; per element one rounding per
 * operation), then per row s' = max|w'|/127 and the codes by the same
 * Philox-keyed stochastic rounding as ref_update_sr (row index n0 + n keys
 * the stream).  The scale factor uses the whole weight's N and K (Nfull),
 * which a slice of rows does not change. */
uint32_t ref_update_muon_sr(int8_t *q, float *s, const float *O, int64_t N, int64_t K,
                            int64_t Nfull, float lr, float wd, uint64_t seed, uint64_t step,
                            int64_t n0) {
    if (step < 1) return ORC_BIT_ARG;
    const double scale = Nfull > K ? sqrt((double)Nfull / (double)K) : 1.0;
    const float a = (float)(1.0 - (double)lr * (double)wd);
    const float st = (float)((double)lr * scale);
    uint32_t status = 0;
    float *w = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            const float wv = s[n] * (float)q[n * K + k];
            w[k] = wv * a - st * O[n * K + k];
        }
        status |= sr_requant_row(w, K, n0 + n, seed, step, q + n * K, &s[n]);
    }
    free(w);
    return status;
}

/* AdamW on a float32 vector (the "aux" optimizer of MuonAuxAdamW for biases
 * and other float parameters): the same per-element arithmetic and host
 * constants as the int8 weights' AdamW (ref_update_sr), without
 * requantization. */
uint32_t ref_adamw_vector(float *p, const float *g, float *m, float *v, int64_t n, float lr,
                          float b1, float b2, float eps, float wd, uint64_t step) {
    if (step < 1) return ORC_BIT_ARG;
    adamw_consts c = adamw_setup(lr, b1, b2, eps, wd, step);
    uint32_t st = 0;
    for (int64_t i = 0; i < n; ++i) {
        p[i] = adamw_elem(&c, p[i], g[i], &m[i], &v[i]);
        if (!isfinite(p[i])) st |= ORC_BIT_NONFINITE;
    }
    return st;
}
