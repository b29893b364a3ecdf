"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports
every entry point that include/qlinear.h declares, and rejects bad
arguments on the host before touching the GPU (no launch happens in these
calls, so they run without a device)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import int8_quantized_act_b200 as ql
from int8_quantized_act_b200 import build as cuda_build

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module")
def L():
    cuda_build.build()
    return ql.lib()


def declared_functions():
    names = []
    for h in sorted(os.listdir(INCLUDE)):
        if h.endswith(".h"):
            text = open(os.path.join(INCLUDE, h)).read()
            names += re.findall(r"QL_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert set(names) >= {"qlinear_quantize_rows", "qlinear_hadamard", "qlinear_fwd",
                          "qlinear_bwd_dx", "qlinear_bwd_dw", "qweight_update_sr",
                          "ql_status_string", "qlinear_workspace_bytes", "qlinear_bwd",
                          "qlinear_bwd_dx_noalloc", "ql_test_wait_timeout", "qlinear_dequantize",
                          "qlinear_codes_bf16", "qlinear_fwd_bf16", "qlinear_fwd_bf16_workspace_bytes"}
    for n in names:
        assert hasattr(L, n), n


def test_every_declared_function_has_a_binding_of_the_same_name():
    """The Python binding mirrors the C ABI name for name, and each binding
    function is exported by the package."""
    for n in declared_functions():
        assert callable(getattr(ql, n, None)), n
        assert n in ql.__all__, n


def test_status_strings(L):
    for code in range(9):
        assert ql.ql_status_string(code).startswith("QL_")
    assert ql.status_flags((1 << ql.QL_ERR_ZERO_ROW) | (1 << ql.QL_ERR_TIMEOUT)) == ["ZERO_ROW", "TIMEOUT"]


def test_workspace_formula(L):
    def a(x):
        return (x + 255) // 256 * 256
    M, N, K = 12000, 7168, 5376
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 128) == base
    assert ql.qlinear_workspace_bytes(M, N, K, 256) == base + a(4 * M * K)
    assert ql.qlinear_workspace_bytes(-1, N, K, 0) == 0


P = ctypes.c_void_p


def fake(addr):
    """A pointer value that is never dereferenced: these calls fail validation."""
    return P(addr)


def test_workspace_grows_by_the_int32_partials_of_long_contractions(L):
    def a(x):
        return (x + 255) // 256 * 256
    limit = ql.QL_MAX_CONTRACTION
    # 1023 blocks of 128 per split: 131,072 -> 2 splits, 400,000 -> 4
    # (200 tokens: more than one 128-row slab, so no extra small-output splits)
    M, K = 200, 256
    for N, splits in ((limit + 1, 2), (400000, 4)):
        base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
        assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * splits * M * K)
        # rotated: the float32 product waits for its second pass
        assert ql.qlinear_workspace_bytes(M, N, K, 128) == base + a(4 * M * K) + a(4 * splits * M * K)
    M, N = 262144, 144         # 2048 blocks -> 3 splits over the tokens
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * 3 * N * K)
    # a small output takes the larger of the two split counts
    M, N = 262144, 48
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * 8 * N * K)
    M, N = 8, 1100000          # 8594 blocks -> 9 splits > 8
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * 9 * M * K)


def test_workspace_small_outputs_reserve_split_partials(L):
    """Outputs of at most 128 rows (dX for few tokens, dW for few output
    features) run as up to 8 contraction splits: room for their partials."""
    def a(x):
        return (x + 255) // 256 * 256
    M, N, K = 17, 7168, 5376
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * 8 * M * K)
    assert ql.qlinear_workspace_bytes(M, N, K, 128) == base + a(4 * M * K) + a(4 * 8 * M * K)
    M, N = 4096, 64
    base = a(M * N) + a(4 * M) + 2 * a(4 * N) + a(8 * N)
    assert ql.qlinear_workspace_bytes(M, N, K, 0) == base + a(4 * 8 * N * K)


def test_bwd_workspace_formula(L):
    def a(x):
        return (x + 255) // 256 * 256
    for (M, N, K, B) in ((12000, 7168, 5376, 128), (17, 144, 512, 256)):
        assert (ql.qlinear_bwd_workspace_bytes(M, N, K, B)
                == ql.qlinear_workspace_bytes(M, N, K, B) + a(M * N) + a(4 * M))


def test_host_validation_returns_before_any_launch(L):
    A = 0x10000  # 16-byte aligned fake address
    # bad dtype / block / flags
    assert L.qlinear_quantize_rows(fake(A), 7, 4, 32, 32, None, 0, 0, fake(A), 32, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.qlinear_quantize_rows(fake(A), 0, 4, 32, 32, None, 3, 0, fake(A), 32, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.qlinear_quantize_rows(fake(A), 0, 4, 32, 32, None, 0, 4, fake(A), 32, fake(A), fake(A), None) == ql.QL_ERR_ARG
    # shapes: cols % 16, cols % block, ldq % 16
    assert L.qlinear_quantize_rows(fake(A), 0, 4, 40, 40, None, 0, 0, fake(A), 48, fake(A), fake(A), None) == ql.QL_ERR_SHAPE
    assert L.qlinear_quantize_rows(fake(A), 0, 4, 48, 48, None, 32, 0, fake(A), 48, fake(A), fake(A), None) == ql.QL_ERR_SHAPE
    assert L.qlinear_quantize_rows(fake(A), 0, 4, 32, 32, None, 0, 0, fake(A), 40, fake(A), fake(A), None) == ql.QL_ERR_SHAPE
    # null and misaligned pointers
    assert L.qlinear_quantize_rows(None, 0, 4, 32, 32, None, 0, 0, fake(A), 32, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.qlinear_quantize_rows(fake(A + 4), 0, 4, 32, 32, None, 0, 0, fake(A), 32, fake(A), fake(A), None) == ql.QL_ERR_ALIGN
    # zero rows: nothing to do
    assert L.qlinear_quantize_rows(None, 0, 0, 32, 32, None, 0, 0, None, 32, None, None, None) == ql.QL_OK
    # forward: contraction limit of the pages, K and N multiples of 16
    big = 131072
    assert L.qlinear_fwd(fake(A), 0, 2, big, fake(A), fake(A), 32, None, 0, fake(A), 0, fake(A), fake(A), fake(A), None) == ql.QL_ERR_UNSUPPORTED
    assert L.qlinear_fwd(fake(A), 0, 2, 40, fake(A), fake(A), 32, None, 0, fake(A), 0, fake(A), fake(A), fake(A), None) == ql.QL_ERR_SHAPE
    assert L.qlinear_fwd(fake(A), 0, 2, 32, fake(A), fake(A), 24, None, 0, fake(A), 0, fake(A), fake(A), fake(A), None) == ql.QL_ERR_SHAPE
    assert L.qlinear_fwd(fake(A), 0, 2, 32, fake(A), fake(A), 32, fake(A + 8), 0, fake(A), 0, fake(A), fake(A), fake(A), None) == ql.QL_ERR_ALIGN
    # backward: workspace too small, contraction limit
    assert L.qlinear_bwd_dx(fake(A), 0, 4, 32, fake(A), fake(A), 32, 0, fake(A), 0, fake(0x100000), 16, fake(A), None) == ql.QL_ERR_SHAPE
    # long backward contractions need the larger workspace of their splits
    need = ql.qlinear_workspace_bytes(4, big, 32, 0)
    assert L.qlinear_bwd_dx(fake(A), 0, 4, big, fake(A), fake(A), 32, 0, fake(A), 0, fake(A), need - 256, fake(A), None) == ql.QL_ERR_SHAPE
    need = ql.qlinear_workspace_bytes(big, 32, 32, 0)
    assert L.qlinear_bwd_dw(fake(A), 0, big, 32, fake(A), fake(A), 32, fake(A), None, fake(A), need - 256, fake(A), None) == ql.QL_ERR_SHAPE
    assert L.qlinear_bwd_dw(fake(A), 0, 4, 32, fake(A), fake(A), 32, fake(A), None, fake(A + 16), 1 << 30, fake(A), None) == ql.QL_ERR_ALIGN
    # hadamard: in place needs the same dtype and pitch
    assert L.qlinear_hadamard(fake(A), 0, 32, fake(A), 1, 32, 4, 32, 16, None) == ql.QL_ERR_ARG
    assert L.qlinear_hadamard(fake(A), 0, 32, fake(A), 0, 32, 4, 32, 0, None) == ql.QL_ERR_ARG


def test_noalloc_checks_arguments_before_capacity(L):
    """qlinear_bwd_dx_noalloc returns qlinear_bwd_dx's code for a bad
    argument or shape even when the sizes exceed its scratch, treats an empty
    output as a no-op, and only then reports the capacity; none of these
    calls reaches the device."""
    A = 0x10000
    f, g = L.qlinear_bwd_dx_noalloc, L.qlinear_bwd_dx
    M, N, K = 12000, 7168, 5376  # workspace far beyond the 32 MiB scratch
    assert ql.qlinear_workspace_bytes(M, N, K, 0) > ql.QL_NOALLOC_SCRATCH_BYTES
    ws = fake(0x100000)
    cases = [
        ((fake(A), 7, M, N, fake(A), fake(A), K, 0, fake(A), 0), ql.QL_ERR_ARG),      # dtype
        ((fake(A), 0, M, N, fake(A), fake(A), K, 3, fake(A), 0), ql.QL_ERR_ARG),      # block
        ((fake(A), 0, M, N, fake(A), fake(A), K + 8, 0, fake(A), 0), ql.QL_ERR_SHAPE),  # K % 16
        ((fake(A), 0, M, N, fake(A), fake(A), K + 16, 32, fake(A), 0), ql.QL_ERR_SHAPE),  # K % B
        ((fake(A), 0, M, N, fake(A), fake(A), K, 0, None, 0), ql.QL_ERR_ARG),         # null dx
    ]
    for args, code in cases:
        assert f(*args, fake(A), None) == code
        assert g(*args, ws, 1 << 40, fake(A), None) == code
    # nothing to compute: no-op, whatever the other sizes
    assert f(fake(A), 0, M, N, fake(A), fake(A), 0, 0, fake(A), 0, fake(A), None) == ql.QL_OK
    assert f(None, 0, 0, 10 ** 9, None, None, 16, 0, None, 0, None, None) == ql.QL_OK
    # valid arguments, too large for the scratch
    assert f(fake(A), 0, M, N, fake(A), fake(A), K, 0, fake(A), 0, fake(A), None) == ql.QL_ERR_UNSUPPORTED


def test_update_validation(L):
    A = 0x10000
    opt = ql._Optim(ql.QL_SGD, 0.1, 0.9, 0.999, 1e-8, 0.5)
    f = L.qweight_update_sr
    assert f(fake(A), fake(A), fake(A), 4, 32, ctypes.byref(opt), None, None, 0, 1, None, fake(A), None) == ql.QL_ERR_ARG
    opt = ql._Optim(ql.QL_ADAMW, 1e-3, 0.9, 1.5, 1e-8, 0.0)
    assert f(fake(A), fake(A), fake(A), 4, 32, ctypes.byref(opt), fake(A), fake(A), 0, 1, None, fake(A), None) == ql.QL_ERR_ARG
    opt = ql._Optim(ql.QL_ADAMW, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert f(fake(A), fake(A), fake(A), 4, 32, ctypes.byref(opt), fake(A), fake(A), 0, 0, None, fake(A), None) == ql.QL_ERR_ARG
    assert f(fake(A), fake(A), fake(A), 4, 40, ctypes.byref(opt), fake(A), fake(A), 0, 1, None, fake(A), None) == ql.QL_ERR_SHAPE
    assert f(fake(A), fake(A), fake(A), 4, 32784, ctypes.byref(opt), fake(A), fake(A), 0, 1, None, fake(A), None) == ql.QL_ERR_UNSUPPORTED
    assert f(fake(A), fake(A), fake(A), 4, 32, ctypes.byref(opt), None, fake(A), 0, 1, None, fake(A), None) == ql.QL_ERR_ARG
    assert f(fake(A + 8), fake(A), fake(A), 4, 32, ctypes.byref(opt), fake(A), fake(A), 0, 1, None, fake(A), None) == ql.QL_ERR_ALIGN


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros((4, 32))
    with pytest.raises(TypeError):
        ql.qlinear_quantize_rows(x, torch.zeros((4, 32), dtype=torch.int8), torch.zeros(4),
                                 torch.zeros(1, dtype=torch.int32))


def test_timeout_hook_validation(L):
    assert L.ql_test_wait_timeout(None, 1000, None) == ql.QL_ERR_ARG
    assert L.ql_test_wait_timeout(fake(0x10000), 0, None) == ql.QL_ERR_ARG
    assert L.ql_test_wait_timeout(fake(0x10000), 10000001, None) == ql.QL_ERR_ARG


def test_divrn_hook_validation(L):
    A = 0x10000
    assert L.ql_test_divrn(fake(A), fake(A), -1, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.ql_test_divrn(None, fake(A), 4, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.ql_test_divrn(fake(A), fake(A), 4, fake(A), None, None) == ql.QL_ERR_ARG
    assert L.ql_test_divrn(None, None, 0, None, None, None) == ql.QL_OK
    assert L.ql_test_sqrtrn(fake(A), -1, fake(A), fake(A), None) == ql.QL_ERR_ARG
    assert L.ql_test_sqrtrn(fake(A), 4, None, fake(A), None) == ql.QL_ERR_ARG
    assert L.ql_test_sqrtrn(None, 0, None, None, None) == ql.QL_OK


def test_dequantize_validation(L):
    A = 0x10000
    f = L.qlinear_dequantize
    assert f(fake(A), 32, fake(A), 4, 32, 3, fake(A), 0, 32, None) == ql.QL_ERR_ARG      # block
    assert f(fake(A), 32, fake(A), 4, 32, 0, fake(A), 7, 32, None) == ql.QL_ERR_ARG      # dtype
    assert f(fake(A), 48, fake(A), 4, 48, 32, fake(A), 0, 48, None) == ql.QL_ERR_SHAPE   # K % B
    assert f(fake(A), 40, fake(A), 4, 40, 0, fake(A), 0, 40, None) == ql.QL_ERR_SHAPE    # K % 16
    assert f(fake(A), 24, fake(A), 4, 32, 0, fake(A), 0, 32, None) == ql.QL_ERR_SHAPE    # ldq < K
    assert f(fake(A + 8), 32, fake(A), 4, 32, 0, fake(A), 0, 32, None) == ql.QL_ERR_ALIGN
    assert f(fake(A), 32, fake(A), 4, 32, 0, fake(A), 1, 36, None) == ql.QL_ERR_ALIGN    # bf16 pitch
    assert f(None, 32, None, 0, 32, 0, None, 0, 32, None) == ql.QL_OK                   # nothing to do


def test_bf16_route_validation_and_workspace(L):
    A = 0x10000
    assert ql.lib().qlinear_fwd_bf16_workspace_bytes(100, 512, ql.QL_BF16, 0) == 0
    assert ql.lib().qlinear_fwd_bf16_workspace_bytes(100, 512, ql.QL_BF16, 128) == 102400
    assert ql.lib().qlinear_fwd_bf16_workspace_bytes(3, 32, ql.QL_F32, 0) == 256
    f = L.qlinear_fwd_bf16
    args = lambda **kw: [kw.get("x", fake(A)), kw.get("xt", 1), kw.get("M", 4), kw.get("K", 64),
                         kw.get("w", fake(A)), fake(A), kw.get("N", 32), None, kw.get("B", 0),
                         kw.get("y", fake(A)), 1, kw.get("ws", None), kw.get("wsb", 0), fake(A), None]
    assert f(*args(B=3)) == ql.QL_ERR_ARG
    assert f(*args(K=40)) == ql.QL_ERR_SHAPE
    assert f(*args(N=24)) == ql.QL_ERR_SHAPE
    assert f(*args(B=128)) == ql.QL_ERR_SHAPE                  # K % B
    assert f(*args(B=32)) == ql.QL_ERR_SHAPE                   # needs a workspace
    assert f(*args(B=32, ws=fake(A + 16), wsb=1 << 20)) == ql.QL_ERR_ALIGN
    assert f(*args(x=fake(A + 8))) == ql.QL_ERR_ALIGN
    assert f(*args(M=0)) == ql.QL_OK
    g = L.qlinear_codes_bf16
    assert g(fake(A), 32, 4, 40, fake(A), 40, None) == ql.QL_ERR_SHAPE
    assert g(fake(A), 32, 4, 32, fake(A), 36, None) == ql.QL_ERR_ALIGN
