"""Python access to the CPU oracle (oracle.c) for the INT8 quantized-training
Linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the CUDA library and its
binding never do.  Every function takes and returns numpy arrays and does
argument marshalling only; all arithmetic is in oracle.c, whose comments cite
the passages each step follows.

Status values are bit masks with the same bit positions as the library's
device status word (``1 << code``): ARG 1<<1, SHAPE 1<<2, ZERO_ROW 1<<4,
NONFINITE 1<<5, UNSUPPORTED 1<<6.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

BIT_ARG = 1 << 1
BIT_SHAPE = 1 << 2
BIT_ZERO_ROW = 1 << 4
BIT_NONFINITE = 1 << 5
BIT_UNSUPPORTED = 1 << 6
REJECT_ZERO_ROWS = 1
MAX_CONTRACTION = 131071

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32
_U64 = ctypes.c_uint64
_F = ctypes.c_float


def _declare(L):
    sigs = {
        "ref_hadamard_scale": (_F, [ctypes.c_int]),
        "ref_hadamard_rows": (_U32, [_P, _I64, _P, _I64, _I64, _I64, ctypes.c_int]),
        "ref_hadamard_matrix_f64": (None, [ctypes.c_int, _P]),
        "ref_quantize_rows": (_U32, [_P, _I64, _I64, _I64, _P, ctypes.c_int, _U32, _P, _I64, _P]),
        "ref_dequantize": (_U32, [_P, _I64, _P, _I64, _I64, ctypes.c_int, _P, _I64]),
        "ref_gemm_nt": (_U32, [_P, _I64, _P, _I64, _I64, _I64, _I64, _P, _I64]),
        "ref_gemm_nn": (_U32, [_P, _I64, _P, _I64, _I64, _I64, _I64, _P, _I64]),
        "ref_gemm_tn": (_U32, [_P, _I64, _P, _I64, _I64, _I64, _I64, _P, _I64]),
        "ref_fwd": (_U32, [_P, _I64, _I64, _P, _P, _I64, _P, ctypes.c_int, _P, _P, _P]),
        "ref_round_bf16": (_F, [_F]),
        "ref_fwd_bf16": (_U32, [_P, _I64, _I64, _P, _P, _I64, _P, ctypes.c_int, _P, _P]),
        "ref_bwd_prep_rows": (_U32, [_P, _I64, _I64, _P, _P, _P]),
        "ref_bwd_prep_cols": (_U32, [_P, _I64, _I64, _P, _P, _P, _P]),
        "ref_bwd_dx": (_U32, [_P, _I64, _I64, _P, _P, _I64, ctypes.c_int, _P, _P, _P]),
        "ref_bwd_dw": (_U32, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P, _P]),
        "ref_philox4x32_10": (None, [_P, _P, _P]),
        "ref_sr_u24": (_U32, [_U64, _U64, _U64]),
        "ref_update_sr": (_U32, [_P, _P, _P, _I64, _I64, ctypes.c_int, _F, _F, _F, _F, _F,
                                 _P, _P, _U64, _U64, _P, _P, _P, _I64]),
        "ref_update_float": (_U32, [_P, _P, _P, _I64, _I64, ctypes.c_int, _F, _F, _F, _F, _F,
                                    _P, _P, _U64, _P, _P, _P, _P]),
        "ref_sr_expectation_enum": (ctypes.c_double, [_F]),
        "ref_exp": (_F, [_F]),
        "ref_fwd_quantized": (_U32, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P]),
        "ref_muon_momentum": (None, [_P, _P, _I64, _F, _P]),
        "ref_newton_schulz5": (None, [_P, _I64, _I64, ctypes.c_int, _P]),
        "ref_update_muon_sr": (_U32, [_P, _P, _P, _I64, _I64, _I64, _F, _F, _U64, _U64, _I64]),
        "ref_adamw_vector": (_U32, [_P, _P, _P, _P, _I64, _F, _F, _F, _F, _F, _U64]),
        "ref_swiglu_h": (None, [_P, _I64, _I64, _I64, _P]),
        "ref_swiglu_quantize": (_U32, [_P, _I64, _I64, _I64, _P, _P]),
        "ref_swiglu_bwd": (None, [_P, _I64, _I64, _I64, _P, _P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i8(a):
    return np.ascontiguousarray(a, dtype=np.int8)


# ---------------------------------------------------------------- rotation
def hadamard_scale(B: int) -> float:
    return float(lib().ref_hadamard_scale(B))


def hadamard_rows(x: np.ndarray, B: int):
    x = _f32(x)
    rows, cols = x.shape
    y = np.empty_like(x)
    st = lib().ref_hadamard_rows(_p(x), cols, _p(y), cols, rows, cols, B)
    return y, st


def dequantize(q: np.ndarray, s: np.ndarray, B: int = 0):
    """(s * q) R row by row: the weight back in floating point and in the
    original basis.  Returns (w float32 [N,K], status)."""
    q, s = _i8(q), _f32(s)
    N, K = q.shape
    w = np.empty((N, K), np.float32)
    st = lib().ref_dequantize(_p(q), K, _p(s), N, K, B, _p(w), K)
    return w, st


def hadamard_matrix(B: int) -> np.ndarray:
    R = np.empty((B, B), np.float64)
    lib().ref_hadamard_matrix_f64(B, _p(R))
    return R


# ---------------------------------------------------------------- quantize
def quantize_rows(x: np.ndarray, B: int = 0, col_scale=None, flags: int = 0):
    x = _f32(x)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty((rows,), np.float32)
    cs = None if col_scale is None else _f32(col_scale)
    st = lib().ref_quantize_rows(_p(x), rows, cols, cols, _p(cs), B, flags, _p(q), cols, _p(s))
    return q, s, st


# ---------------------------------------------------------------- GEMMs
def gemm_nt(A: np.ndarray, B: np.ndarray):
    """out[m,n] = sum_c A[m,c] B[n,c] (int32), status."""
    A, B = _i8(A), _i8(B)
    M, C = A.shape
    N = B.shape[0]
    out = np.empty((M, N), np.int32)
    st = lib().ref_gemm_nt(_p(A), C, _p(B), C, M, N, C, _p(out), N)
    return out, st


def gemm_nn(A: np.ndarray, B: np.ndarray):
    """out[m,n] = sum_c A[m,c] B[c,n] (int32), status."""
    A, B = _i8(A), _i8(B)
    M, C = A.shape
    N = B.shape[1]
    out = np.empty((M, N), np.int32)
    st = lib().ref_gemm_nn(_p(A), C, _p(B), N, M, N, C, _p(out), N)
    return out, st


def gemm_tn(A: np.ndarray, B: np.ndarray):
    """out[m,n] = sum_c A[c,m] B[c,n] (int32), status."""
    A, B = _i8(A), _i8(B)
    C, M = A.shape
    N = B.shape[1]
    out = np.empty((M, N), np.int32)
    st = lib().ref_gemm_tn(_p(A), M, _p(B), N, M, N, C, _p(out), N)
    return out, st


# ---------------------------------------------------------------- layer
def fwd(x, wq, sw, bias=None, B: int = 0):
    """Returns y (fp32 [M,N]), X_q, s_x, status."""
    x, wq, sw = _f32(x), _i8(wq), _f32(sw)
    M, K = x.shape
    N = wq.shape[0]
    b = None if bias is None else _f32(bias)
    y = np.empty((M, N), np.float32)
    xq = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    st = lib().ref_fwd(_p(x), M, K, _p(wq), _p(sw), N, _p(b), B, _p(y), _p(xq), _p(sx))
    return y, xq, sx, st


def fwd_quantized(xq, sx, wq, sw, bias=None):
    """The forward from codes and row scales: returns y (fp32 [M,N]), status."""
    xq, sx, wq, sw = _i8(xq), _f32(sx), _i8(wq), _f32(sw)
    M, K = xq.shape
    N = wq.shape[0]
    b = None if bias is None else _f32(bias)
    y = np.empty((M, N), np.float32)
    st = lib().ref_fwd_quantized(_p(xq), _p(sx), M, K, _p(wq), _p(sw), N, _p(b), _p(y))
    return y, st


def round_bf16(v: float) -> float:
    return float(lib().ref_round_bf16(float(v)))


def fwd_bf16(x, wq, sw, bias=None, B: int = 0):
    """The bf16 route: returns y (fp32 [M,N]), xr = bf16(x R) as fp32, status."""
    x, wq, sw = _f32(x), _i8(wq), _f32(sw)
    M, K = x.shape
    N = wq.shape[0]
    b = None if bias is None else _f32(bias)
    y = np.empty((M, N), np.float32)
    xr = np.empty((M, K), np.float32)
    st = lib().ref_fwd_bf16(_p(x), M, K, _p(wq), _p(sw), N, _p(b), B, _p(y), _p(xr))
    return y, xr, st


def bwd_prep_rows(dy, sw):
    dy, sw = _f32(dy), _f32(sw)
    M, N = dy.shape
    q = np.empty((M, N), np.int8)
    s1 = np.empty((M,), np.float32)
    st = lib().ref_bwd_prep_rows(_p(dy), M, N, _p(sw), _p(q), _p(s1))
    return q, s1, st


def bwd_prep_cols(dy, sx):
    dy, sx = _f32(dy), _f32(sx)
    M, N = dy.shape
    q = np.empty((M, N), np.int8)
    s2 = np.empty((N,), np.float32)
    db = np.empty((N,), np.float32)
    st = lib().ref_bwd_prep_cols(_p(dy), M, N, _p(sx), _p(q), _p(s2), _p(db))
    return q, s2, db, st


def bwd_dx(dy, wq, sw, B: int = 0):
    """Returns dX (fp32 [M,K]), dYq_r, s1, status."""
    dy, wq, sw = _f32(dy), _i8(wq), _f32(sw)
    M, N = dy.shape
    K = wq.shape[1]
    dx = np.empty((M, K), np.float32)
    q = np.empty((M, N), np.int8)
    s1 = np.empty((M,), np.float32)
    st = lib().ref_bwd_dx(_p(dy), M, N, _p(wq), _p(sw), K, B, _p(dx), _p(q), _p(s1))
    return dx, q, s1, st


def bwd_dw(dy, xq, sx):
    """Returns dW (fp32 [N,K]), db, dYq_c, s2, status."""
    dy, xq, sx = _f32(dy), _i8(xq), _f32(sx)
    M, N = dy.shape
    K = xq.shape[1]
    dw = np.empty((N, K), np.float32)
    db = np.empty((N,), np.float32)
    q = np.empty((M, N), np.int8)
    s2 = np.empty((N,), np.float32)
    st = lib().ref_bwd_dw(_p(dy), M, N, _p(xq), _p(sx), K, _p(dw), _p(db), _p(q), _p(s2))
    return dw, db, q, s2, st


# ---------------------------------------------------------------- RNG / update
def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, np.uint32)
    lib().ref_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_u24(seed: int, step: int, e: int) -> int:
    return int(lib().ref_sr_u24(seed, step, e))


def sr_expectation_enum(v: float) -> float:
    return float(lib().ref_sr_expectation_enum(v))


SGD, ADAMW = 0, 1


def update_sr(q, s, grad, kind: int, lr: float, seed: int, step: int,
              m=None, v=None, b1=0.9, b2=0.999, eps=1e-8, wd=0.0,
              g=None, g_m=None, g_v=None, row0: int = 0):
    """One optimizer step with stochastic requantization; returns the new
    (q, s, m, v, g, g_m, g_v, status) as copies (inputs are not modified).
    The arrays hold rows row0.. of the weight (row0 keys the random stream)."""
    q, s, grad = _i8(q).copy(), _f32(s).copy(), _f32(grad)
    N, K = q.shape
    m = None if m is None else _f32(m).copy()
    v = None if v is None else _f32(v).copy()
    g = None if g is None else _f32(g).copy()
    g_m = None if g_m is None else _f32(g_m).copy()
    g_v = None if g_v is None else _f32(g_v).copy()
    st = lib().ref_update_sr(_p(q), _p(s), _p(grad), N, K, kind, lr, b1, b2, eps, wd,
                             _p(m), _p(v), seed, step, _p(g), _p(g_m), _p(g_v), row0)
    return q, s, m, v, g, g_m, g_v, st


def update_float(q, s, grad, kind: int, lr: float, step: int,
                 m=None, v=None, b1=0.9, b2=0.999, eps=1e-8, wd=0.0,
                 g=None, g_m=None, g_v=None):
    """The optimizer step alone, without requantization; returns the updated
    float weights (or directions) [N,K] and the new (m, v, g, g_m, g_v), status."""
    q, s, grad = _i8(q), _f32(s), _f32(grad)
    N, K = q.shape
    m = None if m is None else _f32(m).copy()
    v = None if v is None else _f32(v).copy()
    g = None if g is None else _f32(g).copy()
    g_m = None if g_m is None else _f32(g_m).copy()
    g_v = None if g_v is None else _f32(g_v).copy()
    w = np.empty((N, K), np.float32)
    st = lib().ref_update_float(_p(q), _p(s), _p(grad), N, K, kind, lr, b1, b2, eps, wd,
                                _p(m), _p(v), step, _p(g), _p(g_m), _p(g_v), _p(w))
    return w, m, v, g, g_m, g_v, st


# ---------------------------------------------------------------- SwiGLU gate
def exp(x: float) -> float:
    """e^x in float32 by the oracle's stated method (see oracle.c)."""
    return float(lib().ref_exp(float(x)))


def exp_array(x: np.ndarray) -> np.ndarray:
    f = lib().ref_exp
    x = _f32(x)
    return np.array([f(float(v)) for v in x.ravel()], np.float32).reshape(x.shape)


def swiglu_h(ab: np.ndarray) -> np.ndarray:
    """h = silu(a) * b for ab = [a | b] of shape [M, 2F]; returns h [M, F]."""
    ab = _f32(ab)
    M, F2 = ab.shape
    F = F2 // 2
    h = np.empty((M, F), np.float32)
    lib().ref_swiglu_h(_p(ab), M, F, F2, _p(h))
    return h


def swiglu_quantize(ab: np.ndarray):
    """The second projection's saved input: (h codes [M, F], s_h [M], status)."""
    ab = _f32(ab)
    M, F2 = ab.shape
    F = F2 // 2
    q = np.empty((M, F), np.int8)
    s = np.empty((M,), np.float32)
    st = lib().ref_swiglu_quantize(_p(ab), M, F, F2, _p(q), _p(s))
    return q, s, st


def swiglu_bwd(ab: np.ndarray, dh: np.ndarray) -> np.ndarray:
    """[da | db] [M, 2F] from ab [M, 2F] and dh [M, F]."""
    ab, dh = _f32(ab), _f32(dh)
    M, F2 = ab.shape
    F = F2 // 2
    assert dh.shape == (M, F)
    dab = np.empty((M, F2), np.float32)
    lib().ref_swiglu_bwd(_p(ab), M, F, F2, _p(dh), _p(dab))
    return dab


# ---------------------------------------------------------------- MuonAuxAdamW
def muon_momentum(G, M, beta: float = 0.95):
    """Returns (M', U): the new momentum and the Nesterov-blended update."""
    G = _f32(G)
    M2 = _f32(M).copy()
    U = np.empty_like(G)
    lib().ref_muon_momentum(_p(G), _p(M2), G.size, beta, _p(U))
    return M2, U


def newton_schulz5(U, steps: int = 5) -> np.ndarray:
    """The orthogonalized update NS5(U) in float64 [R, C]."""
    U = _f32(U)
    R, C = U.shape
    O = np.empty((R, C), np.float64)
    lib().ref_newton_schulz5(_p(U), R, C, steps, _p(O))
    return O


def update_muon_sr(q, s, O, lr: float, wd: float, seed: int, step: int, n_full=None,
                   row0: int = 0):
    """One Muon step with stochastic requantization from the float32 update O;
    returns the new (q, s, status) as copies.  n_full: rows of the whole weight
    (for the max(1, N/K)^0.5 factor) when q holds a slice of rows from row0."""
    q, s, O = _i8(q).copy(), _f32(s).copy(), _f32(O)
    N, K = q.shape
    st = lib().ref_update_muon_sr(_p(q), _p(s), _p(O), N, K, N if n_full is None else n_full,
                                  lr, wd, seed, step, row0)
    return q, s, st


def adamw_vector(p, g, m, v, lr: float, step: int, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    """AdamW on a float32 vector; returns new (p, m, v, status)."""
    p, g = _f32(p).copy(), _f32(g)
    m, v = _f32(m).copy(), _f32(v).copy()
    st = lib().ref_adamw_vector(_p(p), _p(g), _p(m), _p(v), p.size, lr, b1, b2, eps, wd, step)
    return p, m, v, st
