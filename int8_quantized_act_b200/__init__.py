"""int8_quantized_act_b200 - INT8 quantized-training Linear layer for B200.

Thin Python binding of the C-ABI library ``libqlinear.so`` (declared in
``include/qlinear.h``).  Each function has the name of the C entry point,
takes torch CUDA tensors, checks that they are CUDA tensors of the expected
dtype and layout, passes their device pointers and sizes, and raises
``QLError`` on a non-zero return code.  Every step of the layer runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing
this package fails loudly if the library has not been built.

Build the library with ``python -m int8_quantized_act_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "QL_OK", "QL_ERR_ARG", "QL_ERR_SHAPE", "QL_ERR_ALIGN", "QL_ERR_ZERO_ROW",
    "QL_ERR_NONFINITE", "QL_ERR_UNSUPPORTED", "QL_ERR_CUDA", "QL_ERR_TIMEOUT",
    "QL_F32", "QL_BF16", "QL_SGD", "QL_ADAMW", "QL_REJECT_ZERO_ROWS",
    "QL_MAX_CONTRACTION", "QLError", "Optim", "lib", "library_path",
    "ql_status_string", "qlinear_workspace_bytes", "qlinear_quantize_rows",
    "qlinear_hadamard", "qlinear_dequantize", "qlinear_codes_bf16", "qlinear_fwd_bf16",
    "qlinear_fwd_bf16_workspace_bytes", "qlinear_fwd", "qlinear_bwd_dx", "qlinear_bwd_dw",
    "qweight_update_sr", "status_flags", "ql_set_gemm_timing_events", "ql_kernel_launches",
    "qlinear_bwd_dx_noalloc", "QL_NOALLOC_SCRATCH_BYTES", "qlinear_bwd",
    "qlinear_bwd_workspace_bytes", "ql_test_wait_timeout", "ql_test_divrn", "ql_test_sqrtrn", "qlinear_fwd_quantized",
    "qlinear_swiglu_quantize", "qlinear_swiglu_bwd", "qweight_muon_workspace_bytes",
    "qweight_muon_orthogonalize", "qweight_update_muon_sr", "qvector_adamw",
]

QL_OK, QL_ERR_ARG, QL_ERR_SHAPE, QL_ERR_ALIGN = 0, 1, 2, 3
QL_ERR_ZERO_ROW, QL_ERR_NONFINITE, QL_ERR_UNSUPPORTED = 4, 5, 6
QL_ERR_CUDA, QL_ERR_TIMEOUT = 7, 8
QL_F32, QL_BF16 = 0, 1
QL_SGD, QL_ADAMW = 0, 1
QL_REJECT_ZERO_ROWS = 1
QL_MAX_CONTRACTION = 131071
QL_NOALLOC_SCRATCH_BYTES = 32 << 20

_NAMES = {
    QL_OK: "OK", QL_ERR_ARG: "ARG", QL_ERR_SHAPE: "SHAPE", QL_ERR_ALIGN: "ALIGN",
    QL_ERR_ZERO_ROW: "ZERO_ROW", QL_ERR_NONFINITE: "NONFINITE",
    QL_ERR_UNSUPPORTED: "UNSUPPORTED", QL_ERR_CUDA: "CUDA", QL_ERR_TIMEOUT: "TIMEOUT",
}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlinear.so")


class QLError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ql_status_string(code)}")


class _Optim(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("lr", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


class _WeightNorm(ctypes.Structure):
    _fields_ = [("g", ctypes.c_void_p), ("g_m", ctypes.c_void_p), ("g_v", ctypes.c_void_p)]


@dataclass
class Optim:
    """Optimizer hyper-parameters of qweight_update_sr (see include/qlinear.h)."""
    kind: int = QL_ADAMW
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlinear.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(
            f"{library_path} is missing: build it with "
            "`python -m int8_quantized_act_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(library_path)
    P, I64, I, U, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint, ctypes.c_float
    L.ql_status_string.restype = ctypes.c_char_p
    L.ql_status_string.argtypes = [I]
    L.qlinear_workspace_bytes.restype = ctypes.c_size_t
    L.qlinear_workspace_bytes.argtypes = [I64, I64, I64, I]
    L.qlinear_quantize_rows.restype = I
    L.qlinear_quantize_rows.argtypes = [P, I, I64, I64, I64, P, I, U, P, I64, P, P, P]
    L.qlinear_hadamard.restype = I
    L.qlinear_hadamard.argtypes = [P, I, I64, P, I, I64, I64, I64, I, P]
    L.qlinear_dequantize.restype = I
    L.qlinear_dequantize.argtypes = [P, I64, P, I64, I64, I, P, I, I64, P]
    L.qlinear_codes_bf16.restype = I
    L.qlinear_codes_bf16.argtypes = [P, I64, I64, I64, P, I64, P]
    L.qlinear_fwd_bf16_workspace_bytes.restype = ctypes.c_size_t
    L.qlinear_fwd_bf16_workspace_bytes.argtypes = [I64, I64, I, I]
    L.qlinear_fwd_bf16.restype = I
    L.qlinear_fwd_bf16.argtypes = [P, I, I64, I64, P, P, I64, P, I, P, I, P, ctypes.c_size_t, P, P]
    L.qlinear_fwd.restype = I
    L.qlinear_fwd.argtypes = [P, I, I64, I64, P, P, I64, P, I, P, I, P, P, P, P]
    L.qlinear_bwd_dx.restype = I
    L.qlinear_bwd_dx.argtypes = [P, I, I64, I64, P, P, I64, I, P, I, P, ctypes.c_size_t, P, P]
    L.qlinear_bwd_dw.restype = I
    L.qlinear_bwd_dw.argtypes = [P, I, I64, I64, P, P, I64, P, P, P, ctypes.c_size_t, P, P]
    L.ql_test_wait_timeout.restype = I
    L.ql_test_wait_timeout.argtypes = [P, ctypes.c_uint32, P]
    L.ql_test_divrn.restype = I
    L.ql_test_divrn.argtypes = [P, P, I64, P, P, P]
    L.ql_test_sqrtrn.restype = I
    L.ql_test_sqrtrn.argtypes = [P, I64, P, P, P]
    L.qlinear_bwd_workspace_bytes.restype = ctypes.c_size_t
    L.qlinear_bwd_workspace_bytes.argtypes = [I64, I64, I64, I]
    L.qlinear_bwd.restype = I
    L.qlinear_bwd.argtypes = [P, I, I64, I64, P, P, P, P, I64, I, P, I, P, P, P,
                              ctypes.c_size_t, P, P]
    L.qlinear_fwd_quantized.restype = I
    L.qlinear_fwd_quantized.argtypes = [P, P, I64, I64, P, P, I64, P, P, I, P, P]
    L.qlinear_swiglu_quantize.restype = I
    L.qlinear_swiglu_quantize.argtypes = [P, I, I64, I64, I64, P, I64, P, P, P]
    L.qlinear_swiglu_bwd.restype = I
    L.qlinear_swiglu_bwd.argtypes = [P, I, I64, P, I, I64, I64, P, I, P]
    L.qweight_muon_workspace_bytes.restype = ctypes.c_size_t
    L.qweight_muon_workspace_bytes.argtypes = [I64, I64]
    L.qweight_muon_orthogonalize.restype = I
    L.qweight_muon_orthogonalize.argtypes = [P, P, I64, I64, F, I, P, P, ctypes.c_size_t, P, P]
    L.qweight_update_muon_sr.restype = I
    L.qweight_update_muon_sr.argtypes = [P, P, P, I64, I64, F, F, ctypes.c_uint64,
                                         ctypes.c_uint64, P, P]
    L.qvector_adamw.restype = I
    L.qvector_adamw.argtypes = [P, P, P, P, I64, ctypes.POINTER(_Optim), ctypes.c_uint64, P, P]
    L.qlinear_bwd_dx_noalloc.restype = I
    L.qlinear_bwd_dx_noalloc.argtypes = [P, I, I64, I64, P, P, I64, I, P, I, P, P]
    L.ql_set_gemm_timing_events.restype = None
    L.ql_set_gemm_timing_events.argtypes = [ctypes.POINTER(ctypes.c_void_p),
                                            ctypes.POINTER(ctypes.c_void_p), I]
    L.ql_kernel_launches.restype = ctypes.c_uint64
    L.ql_kernel_launches.argtypes = []
    L.qweight_update_sr.restype = I
    L.qweight_update_sr.argtypes = [P, P, P, I64, I64, ctypes.POINTER(_Optim), P, P,
                                    ctypes.c_uint64, ctypes.c_uint64,
                                    ctypes.POINTER(_WeightNorm), P, P]
    _lib = L
    return L


# ------------------------------------------------------------------ helpers
def _dtype_code(t: torch.Tensor, what: str) -> int:
    if t.dtype == torch.float32:
        return QL_F32
    if t.dtype == torch.bfloat16:
        return QL_BF16
    raise TypeError(f"{what}: expected float32 or bfloat16, got {t.dtype}")


def _dev(t: Optional[torch.Tensor], what: str, dtype=None):
    """Device pointer of a CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what}: expected a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _rowmajor(t: torch.Tensor, what: str) -> int:
    """Leading dimension of a 2-D tensor whose rows are contiguous."""
    if t.dim() != 2 or (t.size(1) > 1 and t.stride(1) != 1):
        raise ValueError(f"{what}: expected a 2-D tensor with contiguous rows")
    return t.stride(0) if t.size(0) > 1 else max(t.stride(0), t.size(1))


def _contig(t: Optional[torch.Tensor], what: str):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous tensor")


def _fits(t: Optional[torch.Tensor], rows: int, cols: int, what: str, exact_cols: bool):
    """A 2-D operand must hold `rows` rows of `cols` columns: at least `rows`
    rows and exactly `cols` columns (operands the library reads with their
    row length as the leading dimension) or at least `cols` (operands passed
    with their own leading dimension).  The C ABI sees only pointers, so this
    is the one place where a short buffer can be refused before a kernel
    reads or writes past it.  Absent or empty operands are left to the
    library."""
    if t is None or rows == 0 or cols == 0:
        return
    ok = t.dim() == 2 and t.size(0) >= rows and (
        t.size(1) == cols if exact_cols else t.size(1) >= cols)
    if not ok:
        want = f"[>={rows}, {cols}]" if exact_cols else f"[>={rows}, >={cols}]"
        raise ValueError(f"{what}: expected a 2-D tensor of shape {want}, got {list(t.shape)}")


def _holds(t: Optional[torch.Tensor], n: int, what: str):
    """A vector operand must have at least n elements (absent: left to the library)."""
    if t is not None and n > 0 and t.numel() < n:
        raise ValueError(f"{what}: expected at least {n} elements, got {t.numel()}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(code: int, where: str):
    if code != QL_OK:
        raise QLError(code, where)


def ql_status_string(code: int) -> str:
    return lib().ql_status_string(int(code)).decode()


def status_flags(word: int) -> list:
    """Names of the status bits set in a device status word."""
    return [name for code, name in _NAMES.items() if code and (int(word) >> code) & 1]


def qlinear_workspace_bytes(M: int, N: int, K: int, hadamard_block: int = 0) -> int:
    return int(lib().qlinear_workspace_bytes(M, N, K, hadamard_block))


# ------------------------------------------------------------------ entry points
def qlinear_quantize_rows(x, q, row_scale, status, col_scale=None, hadamard_block: int = 0,
                          flags: int = 0, stream=None):
    """q, row_scale <- per-row int8 quantization of x (optionally x*col_scale,
    rotated by the block-Hadamard of width hadamard_block)."""
    rows, cols = x.shape
    _fits(q, rows, cols, "q", exact_cols=False)
    _contig(row_scale, "row_scale")
    _contig(col_scale, "col_scale")
    _holds(row_scale, rows, "row_scale")
    _holds(col_scale, cols, "col_scale")
    _holds(status, 1, "status")
    code = lib().qlinear_quantize_rows(
        _dev(x, "x"), _dtype_code(x, "x"), rows, cols, _rowmajor(x, "x"),
        _dev(col_scale, "col_scale", torch.float32), hadamard_block, flags,
        _dev(q, "q", torch.int8), _rowmajor(q, "q"), _dev(row_scale, "row_scale", torch.float32),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_quantize_rows")


def qlinear_hadamard(x, y, hadamard_block: int, stream=None):
    """y <- x R (R = block-Hadamard / sqrt(block)); y may be x."""
    rows, cols = x.shape
    if tuple(y.shape) != (rows, cols):
        raise ValueError("qlinear_hadamard: x and y shapes differ")
    code = lib().qlinear_hadamard(
        _dev(x, "x"), _dtype_code(x, "x"), _rowmajor(x, "x"), _dev(y, "y"), _dtype_code(y, "y"),
        _rowmajor(y, "y"), rows, cols, hadamard_block, _stream(stream))
    _check(code, "qlinear_hadamard")


def qlinear_dequantize(wq, sw, hadamard_block: int, w, stream=None):
    """w <- (s_w * wq) R: the weight in floating point, back in the original basis."""
    N, K = wq.shape
    if tuple(w.shape) != (N, K):
        raise ValueError("qlinear_dequantize: wq and w shapes differ")
    _contig(sw, "sw")
    _holds(sw, N, "sw")
    code = lib().qlinear_dequantize(
        _dev(wq, "wq", torch.int8), _rowmajor(wq, "wq"), _dev(sw, "sw", torch.float32), N, K,
        hadamard_block, _dev(w, "w"), _dtype_code(w, "w"), _rowmajor(w, "w"), _stream(stream))
    _check(code, "qlinear_dequantize")


def qlinear_codes_bf16(wq, out, stream=None):
    """out <- the int8 codes of wq as bf16 (exact)."""
    N, K = wq.shape
    if tuple(out.shape) != (N, K) or out.dtype != torch.bfloat16:
        raise ValueError("qlinear_codes_bf16: out must be a bf16 tensor shaped like wq")
    code = lib().qlinear_codes_bf16(_dev(wq, "wq", torch.int8), _rowmajor(wq, "wq"), N, K,
                                    _dev(out, "out"), _rowmajor(out, "out"), _stream(stream))
    _check(code, "qlinear_codes_bf16")


def qlinear_fwd_bf16_workspace_bytes(M: int, K: int, x_dtype, hadamard_block: int) -> int:
    xt = QL_BF16 if x_dtype == torch.bfloat16 else QL_F32
    return int(lib().qlinear_fwd_bf16_workspace_bytes(M, K, xt, hadamard_block))


def qlinear_fwd_bf16(x, wq_bf16, sw, bias, hadamard_block: int, y, ws, status, stream=None):
    """y <- the bf16 route of the forward: bf16(x R) times the bf16 codes on the
    tensor cores, times s_w, plus bias (no activation quantization)."""
    M, K = x.shape
    N = wq_bf16.shape[0]
    for t, n in ((x, "x"), (wq_bf16, "wq_bf16"), (sw, "sw"), (bias, "bias"), (y, "y")):
        _contig(t, n)
    _fits(wq_bf16, N, K, "wq_bf16", exact_cols=True)
    _fits(y, M, N, "y", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(bias, N, "bias")
    _holds(status, 1, "status")
    code = lib().qlinear_fwd_bf16(
        _dev(x, "x"), _dtype_code(x, "x"), M, K, _dev(wq_bf16, "wq_bf16", torch.bfloat16),
        _dev(sw, "sw", torch.float32), N, _dev(bias, "bias", torch.float32), hadamard_block,
        _dev(y, "y"), _dtype_code(y, "y"), _dev(ws, "ws"),
        0 if ws is None else ws.numel() * ws.element_size(), _dev(status, "status", torch.int32),
        _stream(stream))
    _check(code, "qlinear_fwd_bf16")


def qlinear_fwd(x, wq, sw, bias, hadamard_block: int, y, xq_saved, sx_saved, status,
                stream=None):
    """y <- forward of the layer; xq_saved, sx_saved <- the int8 input for backward."""
    M, K = x.shape
    N = wq.shape[0]
    for t, n in ((x, "x"), (wq, "wq"), (sw, "sw"), (bias, "bias"), (y, "y"),
                 (xq_saved, "xq_saved"), (sx_saved, "sx_saved")):
        _contig(t, n)
    _fits(wq, N, K, "wq", exact_cols=True)
    _fits(y, M, N, "y", exact_cols=True)
    _fits(xq_saved, M, K, "xq_saved", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(bias, N, "bias")
    _holds(sx_saved, M, "sx_saved")
    _holds(status, 1, "status")
    code = lib().qlinear_fwd(
        _dev(x, "x"), _dtype_code(x, "x"), M, K, _dev(wq, "wq", torch.int8),
        _dev(sw, "sw", torch.float32), N, _dev(bias, "bias", torch.float32), hadamard_block,
        _dev(y, "y"), _dtype_code(y, "y"), _dev(xq_saved, "xq_saved", torch.int8),
        _dev(sx_saved, "sx_saved", torch.float32), _dev(status, "status", torch.int32),
        _stream(stream))
    _check(code, "qlinear_fwd")


def qlinear_fwd_quantized(xq, sx, wq, sw, bias, y, status, stream=None):
    """y <- forward of the layer from an input already quantized (codes xq,
    row scales sx), e.g. by qlinear_swiglu_quantize."""
    M, K = xq.shape
    N = wq.shape[0]
    for t, n in ((xq, "xq"), (sx, "sx"), (wq, "wq"), (sw, "sw"), (bias, "bias"), (y, "y")):
        _contig(t, n)
    _fits(wq, N, K, "wq", exact_cols=True)
    _fits(y, M, N, "y", exact_cols=True)
    _holds(sx, M, "sx")
    _holds(sw, N, "sw")
    _holds(bias, N, "bias")
    _holds(status, 1, "status")
    code = lib().qlinear_fwd_quantized(
        _dev(xq, "xq", torch.int8), _dev(sx, "sx", torch.float32), M, K,
        _dev(wq, "wq", torch.int8), _dev(sw, "sw", torch.float32), N,
        _dev(bias, "bias", torch.float32), _dev(y, "y"), _dtype_code(y, "y"),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_fwd_quantized")


def qlinear_swiglu_quantize(ab, hq, sh, status, stream=None):
    """hq, sh <- per-row quantization of h = silu(a) * b, ab = [a | b] [M, 2F]."""
    M, F2 = ab.shape
    F = F2 // 2
    _fits(hq, M, F, "hq", exact_cols=False)
    _holds(sh, M, "sh")
    _holds(status, 1, "status")
    code = lib().qlinear_swiglu_quantize(
        _dev(ab, "ab"), _dtype_code(ab, "ab"), M, F, _rowmajor(ab, "ab"),
        _dev(hq, "hq", torch.int8), _rowmajor(hq, "hq"), _dev(sh, "sh", torch.float32),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_swiglu_quantize")


def qlinear_swiglu_bwd(ab, dh, dab, stream=None):
    """dab = [da | db] [M, 2F] <- the gate's backward from ab [M, 2F] and dh [M, F]."""
    M, F2 = ab.shape
    F = F2 // 2
    for t, n in ((dh, "dh"), (dab, "dab")):
        _contig(t, n)
    _fits(dh, M, F, "dh", exact_cols=True)
    _fits(dab, M, F2, "dab", exact_cols=True)
    code = lib().qlinear_swiglu_bwd(
        _dev(ab, "ab"), _dtype_code(ab, "ab"), _rowmajor(ab, "ab"), _dev(dh, "dh"),
        _dtype_code(dh, "dh"), M, F, _dev(dab, "dab"), _dtype_code(dab, "dab"),
        _stream(stream))
    _check(code, "qlinear_swiglu_bwd")


def qweight_muon_workspace_bytes(N: int, K: int) -> int:
    return int(lib().qweight_muon_workspace_bytes(N, K))


def qweight_muon_orthogonalize(grad, mom, O, ws, status, momentum: float = 0.95,
                               ns_steps: int = 5, stream=None):
    """mom <- beta*mom + (1-beta)*grad; O (bf16 [N, K]) <- Newton-Schulz of
    the Nesterov-blended update (the Muon direction)."""
    N, K = grad.shape
    for t, n in ((grad, "grad"), (mom, "mom"), (O, "O")):
        _contig(t, n)
    _fits(mom, N, K, "mom", exact_cols=True)
    _fits(O, N, K, "O", exact_cols=True)
    _holds(ws, qweight_muon_workspace_bytes(N, K), "ws")
    _holds(status, 1, "status")
    code = lib().qweight_muon_orthogonalize(
        _dev(grad, "grad", torch.float32), _dev(mom, "mom", torch.float32), N, K, momentum,
        ns_steps, _dev(O, "O", torch.bfloat16), _dev(ws, "ws", torch.uint8), ws.numel(),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qweight_muon_orthogonalize")


def qweight_update_muon_sr(wq, sw, O, lr: float, weight_decay: float, seed: int, step: int,
                           status, stream=None):
    """The Muon step of the int8 weight from O, with stochastic requantization, in place."""
    N, K = wq.shape
    for t, n in ((wq, "wq"), (sw, "sw"), (O, "O")):
        _contig(t, n)
    _fits(O, N, K, "O", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(status, 1, "status")
    code = lib().qweight_update_muon_sr(
        _dev(wq, "wq", torch.int8), _dev(sw, "sw", torch.float32), _dev(O, "O", torch.bfloat16),
        N, K, lr, weight_decay, seed, step, _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qweight_update_muon_sr")


def qvector_adamw(p, g, m, v, opt: Optim, step: int, status, stream=None):
    """AdamW on a float32 vector (biases and other float parameters), in place."""
    n = p.numel()
    for t, nm in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
        _contig(t, nm)
        _holds(t, n, nm)
    _holds(status, 1, "status")
    o = _Optim(opt.kind, opt.lr, opt.beta1, opt.beta2, opt.eps, opt.weight_decay)
    code = lib().qvector_adamw(
        _dev(p, "p", torch.float32), _dev(g, "g", torch.float32), _dev(m, "m", torch.float32),
        _dev(v, "v", torch.float32), n, ctypes.byref(o), step,
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qvector_adamw")


def qlinear_bwd_dx(dy, wq, sw, hadamard_block: int, dx, ws, status, stream=None):
    """dx <- input gradient from dY and the int8 weight."""
    M, N = dy.shape
    K = wq.shape[1]
    for t, n in ((dy, "dy"), (wq, "wq"), (sw, "sw"), (dx, "dx")):
        _contig(t, n)
    _fits(wq, N, K, "wq", exact_cols=True)
    _fits(dx, M, K, "dx", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(status, 1, "status")
    code = lib().qlinear_bwd_dx(
        _dev(dy, "dy"), _dtype_code(dy, "dy"), M, N, _dev(wq, "wq", torch.int8),
        _dev(sw, "sw", torch.float32), K, hadamard_block, _dev(dx, "dx"), _dtype_code(dx, "dx"),
        _dev(ws, "ws", torch.uint8), ws.numel(), _dev(status, "status", torch.int32),
        _stream(stream))
    _check(code, "qlinear_bwd_dx")


def qlinear_bwd_workspace_bytes(M: int, N: int, K: int, hadamard_block: int = 0) -> int:
    return int(lib().qlinear_bwd_workspace_bytes(M, N, K, hadamard_block))


def qlinear_bwd(dy, wq, sw, xq, sx, hadamard_block: int, dx, dw, db, ws, status, stream=None):
    """dx, dw, db <- both backward products with one shared preparation of dY
    (ws: qlinear_bwd_workspace_bytes bytes)."""
    M, N = dy.shape
    K = wq.shape[1]
    for t, n in ((dy, "dy"), (wq, "wq"), (sw, "sw"), (xq, "xq"), (sx, "sx"), (dx, "dx"),
                 (dw, "dw"), (db, "db")):
        _contig(t, n)
    _fits(wq, N, K, "wq", exact_cols=True)
    _fits(xq, M, K, "xq", exact_cols=True)
    _fits(dx, M, K, "dx", exact_cols=True)
    _fits(dw, N, K, "dw", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(sx, M, "sx")
    _holds(db, N, "db")
    _holds(status, 1, "status")
    code = lib().qlinear_bwd(
        _dev(dy, "dy"), _dtype_code(dy, "dy"), M, N, _dev(wq, "wq", torch.int8),
        _dev(sw, "sw", torch.float32), _dev(xq, "xq", torch.int8), _dev(sx, "sx", torch.float32),
        K, hadamard_block, _dev(dx, "dx"), _dtype_code(dx, "dx"), _dev(dw, "dw", torch.float32),
        _dev(db, "db", torch.float32), _dev(ws, "ws", torch.uint8), ws.numel(),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_bwd")


def qlinear_bwd_dx_noalloc(dy, wq, sw, hadamard_block: int, dx, status, stream=None):
    """qlinear_bwd_dx for callers that cannot allocate device memory: no
    workspace argument; the library's own fixed scratch (QL_NOALLOC_SCRATCH_BYTES)
    is used instead, shared by all calls in the process (calls that may
    overlap on the GPU race on it).  Sizes that need more scratch raise
    QLError(QL_ERR_UNSUPPORTED)."""
    M, N = dy.shape
    K = wq.shape[1]
    for t, n in ((dy, "dy"), (wq, "wq"), (sw, "sw"), (dx, "dx")):
        _contig(t, n)
    _fits(wq, N, K, "wq", exact_cols=True)
    _fits(dx, M, K, "dx", exact_cols=True)
    _holds(sw, N, "sw")
    _holds(status, 1, "status")
    code = lib().qlinear_bwd_dx_noalloc(
        _dev(dy, "dy"), _dtype_code(dy, "dy"), M, N, _dev(wq, "wq", torch.int8),
        _dev(sw, "sw", torch.float32), K, hadamard_block, _dev(dx, "dx"), _dtype_code(dx, "dx"),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_bwd_dx_noalloc")


def qlinear_bwd_dw(dy, xq, sx, dw, db, ws, status, stream=None):
    """dw (float32 [N,K]), db (float32 [N] or None) <- weight/bias gradients."""
    M, N = dy.shape
    K = xq.shape[1]
    for t, n in ((dy, "dy"), (xq, "xq"), (sx, "sx"), (dw, "dw"), (db, "db")):
        _contig(t, n)
    _fits(xq, M, K, "xq", exact_cols=True)
    _fits(dw, N, K, "dw", exact_cols=True)
    _holds(sx, M, "sx")
    _holds(db, N, "db")
    _holds(status, 1, "status")
    code = lib().qlinear_bwd_dw(
        _dev(dy, "dy"), _dtype_code(dy, "dy"), M, N, _dev(xq, "xq", torch.int8),
        _dev(sx, "sx", torch.float32), K, _dev(dw, "dw", torch.float32),
        _dev(db, "db", torch.float32), _dev(ws, "ws", torch.uint8), ws.numel(),
        _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qlinear_bwd_dw")


def qweight_update_sr(wq, sw, grad, opt: Optim, m, v, seed: int, step: int, status,
                      g=None, g_m=None, g_v=None, stream=None):
    """One optimizer step of the int8 weight with stochastic requantization,
    in place (wq, sw, m, v and, for weight norm, g, g_m, g_v)."""
    N, K = wq.shape
    for t, n in ((wq, "wq"), (sw, "sw"), (grad, "grad"), (m, "m"), (v, "v"), (g, "g"),
                 (g_m, "g_m"), (g_v, "g_v")):
        _contig(t, n)
    for t, n in ((grad, "grad"), (m, "m"), (v, "v")):
        _fits(t, N, K, n, exact_cols=True)
    for t, n in ((sw, "sw"), (g, "g"), (g_m, "g_m"), (g_v, "g_v")):
        _holds(t, N, n)
    _holds(status, 1, "status")
    o = _Optim(int(opt.kind), float(opt.lr), float(opt.beta1), float(opt.beta2),
               float(opt.eps), float(opt.weight_decay))
    wn = None
    if g is not None:
        wn = ctypes.pointer(_WeightNorm(_dev(g, "g", torch.float32), _dev(g_m, "g_m", torch.float32),
                                        _dev(g_v, "g_v", torch.float32)))
    code = lib().qweight_update_sr(
        _dev(wq, "wq", torch.int8), _dev(sw, "sw", torch.float32), _dev(grad, "grad", torch.float32),
        N, K, ctypes.byref(o), _dev(m, "m", torch.float32), _dev(v, "v", torch.float32),
        int(seed), int(step), wn, _dev(status, "status", torch.int32), _stream(stream))
    _check(code, "qweight_update_sr")


def ql_set_gemm_timing_events(pairs=()):
    """Record each (before, after) pair of torch.cuda.Event objects around the
    next int8 GEMM launches of this thread, in order (empty: stop).  Each
    event must have been recorded once before (torch creates the underlying
    CUDA event lazily)."""
    n = len(pairs)
    b = (ctypes.c_void_p * max(n, 1))(*[p[0].cuda_event for p in pairs])
    a = (ctypes.c_void_p * max(n, 1))(*[p[1].cuda_event for p in pairs])
    lib().ql_set_gemm_timing_events(b, a, n)


def ql_kernel_launches() -> int:
    """CUDA kernels launched by the library in this process so far."""
    return int(lib().ql_kernel_launches())


def ql_test_wait_timeout(status, limit_us: int, stream=None):
    """Failure-detection check (include/qlinear_testing.h): a kernel waits on
    a barrier that nothing completes; its bounded wait gives up after
    limit_us and sets the QL_ERR_TIMEOUT bit in `status`."""
    _check(lib().ql_test_wait_timeout(_dev(status, "status", torch.int32), int(limit_us),
                                      _stream(stream)), "ql_test_wait_timeout")


def ql_test_divrn(a, d, q, y, stream=None):
    """The SwiGLU gate's float32 division steps (include/qlinear_testing.h)
    on float32 device vectors: q = a / d and y = 1 / d elementwise."""
    n = a.numel()
    for t, what in ((d, "d"), (q, "q"), (y, "y")):
        if t.numel() != n:
            raise ValueError(f"ql_test_divrn: {what} has {t.numel()} values, a has {n}")
    _check(lib().ql_test_divrn(_dev(a, "a", torch.float32), _dev(d, "d", torch.float32), n,
                               _dev(q, "q", torch.float32), _dev(y, "y", torch.float32),
                               _stream(stream)), "ql_test_divrn")


def ql_test_sqrtrn(v, s_plain, s_refined, stream=None):
    """The optimizer updates' float32 square-root steps
    (include/qlinear_testing.h) on a float32 device vector: the plain and the
    refined form of sqrt(v), elementwise."""
    n = v.numel()
    for t, what in ((s_plain, "s_plain"), (s_refined, "s_refined")):
        if t.numel() != n:
            raise ValueError(f"ql_test_sqrtrn: {what} has {t.numel()} values, v has {n}")
    _check(lib().ql_test_sqrtrn(_dev(v, "v", torch.float32), n,
                                _dev(s_plain, "s_plain", torch.float32),
                                _dev(s_refined, "s_refined", torch.float32), _stream(stream)),
           "ql_test_sqrtrn")
