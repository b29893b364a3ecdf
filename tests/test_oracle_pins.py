"""Pins of the CPU oracle against facts that do not come from the oracle itself:
values printed on the pages, closed forms, library routines (scipy's
Hadamard matrix, numpy integer matmul, numpy's round-half-even, cuRAND's
host Philox4x32-10, torch.optim and torch autograd), brute force on tiny
inputs, and invariants of the method.  CPU only.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.txt")


def golden() -> dict:
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, value = line.split("|")[0].split()
        out[name] = value
    return out


# --------------------------------------------------------------------------
# Block-Hadamard rotation
# --------------------------------------------------------------------------

def _rotation_fp32(B: int) -> np.ndarray:
    R, st = oracle.hadamard_rows(np.eye(B, dtype=np.float32), B)
    assert st == 0
    return R


def test_orthogonality_matches_page_value():
    """OneTrainer PR #1681 item 3 prints 5.96e-08 for the fp32 buffer; the
    required bound is 1e-7 for every block size."""
    page = float(golden()["hadamard_orthogonality_fp32_B128"])
    R = torch.from_numpy(_rotation_fp32(128))
    err = (R @ R.T - torch.eye(128)).abs().max().item()
    assert f"{err:.2e}" == f"{page:.2e}"
    for B in (2, 4, 8, 16, 32, 64, 128, 256):
        R = torch.from_numpy(_rotation_fp32(B)).double()
        assert (R @ R.T - torch.eye(B, dtype=torch.float64)).abs().max().item() <= 1e-7


@pytest.mark.parametrize("B", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_equals_sylvester_matrix(B):
    """The butterfly form equals x @ H_B / sqrt(B), H_B from scipy (Sylvester)."""
    x = workloads.normal((5, 3 * B), 1.0, 100 + B)
    y, st = oracle.hadamard_rows(x, B)
    assert st == 0
    H = scipy.linalg.hadamard(B).astype(np.float64) / math.sqrt(B)
    ref = np.concatenate([x[:, i * B:(i + 1) * B].astype(np.float64) @ H for i in range(3)], 1)
    assert np.abs(y - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
    Rd = oracle.hadamard_matrix(B)
    assert np.array_equal(Rd, H)


def test_fwht_is_an_involution():
    """H_B / sqrt(B) is symmetric and orthogonal, so applying it twice is I."""
    x = workloads.normal((7, 512), 1.0, 7)
    for B in (2, 16, 128, 256):
        y, _ = oracle.hadamard_rows(x, B)
        z, _ = oracle.hadamard_rows(y, B)
        assert np.abs(z - x).max() <= 1e-5


def test_rotation_identity_rotating_x_not_unrotating_w():
    """(xR)(WR)^T == x W^T  (OneTrainer PR #1681 item 2 / Summary b)."""
    x = workloads.normal((16, 384), 1.0, 1)
    W = workloads.normal((24, 384), 0.02, 2)
    xr, _ = oracle.hadamard_rows(x, 128)
    wr, _ = oracle.hadamard_rows(W, 128)
    lhs = xr.astype(np.float64) @ wr.astype(np.float64).T
    rhs = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) <= 1e-6


def test_hadamard_rejects_bad_blocks():
    x = np.zeros((2, 96), np.float32)
    assert oracle.hadamard_rows(x, 64)[1] == oracle.BIT_SHAPE  # 96 % 64 != 0
    assert oracle.hadamard_rows(x, 3)[1] == oracle.BIT_SHAPE
    assert oracle.quantize_rows(x, B=3)[2] == oracle.BIT_ARG
    assert oracle.quantize_rows(x, B=512)[2] == oracle.BIT_ARG
    assert oracle.quantize_rows(x, B=64)[2] == oracle.BIT_SHAPE


# --------------------------------------------------------------------------
# Per-row INT8 quantization
# --------------------------------------------------------------------------

def test_quant_exact_multiples_round_trip():
    """Rows s0*q with s0 a power of two and max |q| = 127 quantize to q, s0."""
    rng = np.random.Generator(np.random.PCG64(3))
    q = rng.integers(-127, 128, size=(9, 64)).astype(np.int8)
    q[:, 5] = np.where(np.arange(9) % 2 == 0, 127, -127)
    s0 = (2.0 ** -rng.integers(0, 12, size=9)).astype(np.float32)
    x = q.astype(np.float32) * s0[:, None]
    qq, s, st = oracle.quantize_rows(x)
    assert st == 0
    assert np.array_equal(qq, q)
    assert np.array_equal(s, s0)


def test_quant_ties_round_to_even():
    """With amax = 127 the codes are numpy's round-half-to-even of x."""
    vals = np.array([127.0, -127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 126.5,
                     -126.5, 4.4999995, 0.0, 64.5, 65.5, -1.5], np.float32)
    x = np.tile(vals, (2, 1))
    q, s, st = oracle.quantize_rows(x)
    assert st == 0 and np.all(s == np.float32(1.0))
    assert np.array_equal(q[0], np.rint(vals).astype(np.int8))


def test_quant_error_bound_and_extremes():
    """|t - s q| <= s/2 (+1 ulp), the amax element maps to +-127, |q| <= 127,
    signs agree, and s = amax / 127."""
    d = workloads.tiny_layer()
    for x in (d["x"], d["w"], workloads.normal((33, 512), 3.0, 9)):
        q, s, st = oracle.quantize_rows(x)
        assert st == 0
        amax = np.abs(x).max(1)
        assert np.array_equal(s, (amax / np.float32(127)).astype(np.float32))
        err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[:, None])
        assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-6))
        idx = np.abs(x).argmax(1)
        assert np.array_equal(np.abs(q[np.arange(len(q)), idx]), np.full(len(q), 127, np.int8))
        assert np.abs(q.astype(np.int32)).max() <= 127
        assert np.all((np.sign(q) == np.sign(x)) | (q == 0))


def test_quant_zero_rows():
    """Zero rows: s = 0, codes 0; flagged only when the caller rejects them
    (zero directions are rejected, masked rows are legal)."""
    x = workloads.normal((4, 32), 1.0, 4)
    x[2] = 0.0
    q, s, st = oracle.quantize_rows(x)
    assert st == 0 and s[2] == 0 and not q[2].any()
    q2, s2, st2 = oracle.quantize_rows(x, flags=oracle.REJECT_ZERO_ROWS)
    assert st2 == oracle.BIT_ZERO_ROW
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_quant_nonfinite_flag():
    x = workloads.normal((3, 32), 1.0, 5)
    x[1, 7] = np.nan
    assert oracle.quantize_rows(x)[2] & oracle.BIT_NONFINITE
    x[1, 7] = np.inf
    assert oracle.quantize_rows(x)[2] & oracle.BIT_NONFINITE


def test_quant_composes_with_col_scale_and_rotation():
    x = workloads.normal((6, 256), 1.0, 6)
    c = workloads.uniform((256,), 0.1, 3.0, 7)
    a = oracle.quantize_rows(x, col_scale=c)
    b = oracle.quantize_rows(x * c)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    xr, _ = oracle.hadamard_rows(x, 64)
    a = oracle.quantize_rows(x, B=64)
    b = oracle.quantize_rows(xr)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# --------------------------------------------------------------------------
# Dequantization back to the original basis
# --------------------------------------------------------------------------

def test_dequantize_exact_multiples_round_trip():
    """Rows s0*q (s0 a power of two, max |q| = 127) quantize to (q, s0) and
    dequantize back to exactly the same rows."""
    rng = np.random.Generator(np.random.PCG64(21))
    q = rng.integers(-127, 128, size=(7, 96)).astype(np.int8)
    q[:, 3] = 127
    s0 = (2.0 ** -rng.integers(0, 10, size=7)).astype(np.float32)
    x = q.astype(np.float32) * s0[:, None]
    qq, s, _ = oracle.quantize_rows(x)
    w, st = oracle.dequantize(qq, s)
    assert st == 0 and np.array_equal(w, x)


@pytest.mark.parametrize("B", [2, 16, 128, 256])
def test_dequantize_unrotates_against_scipy_hadamard(B):
    """(s q) R against float64 (s q) @ blockdiag(scipy H_B)/sqrt(B): within a
    few float32 ulps of the row's magnitude (log2 B butterfly roundings)."""
    K = 2 * max(B, 64)
    rng = np.random.Generator(np.random.PCG64(B))
    q = rng.integers(-127, 128, size=(5, K)).astype(np.int8)
    s = rng.uniform(1e-4, 1e-2, size=5).astype(np.float32)
    w, st = oracle.dequantize(q, s, B)
    assert st == 0
    H = scipy.linalg.hadamard(B).astype(np.float64) / math.sqrt(B)
    deq = q.astype(np.float64) * s.astype(np.float64)[:, None]
    ref = (deq.reshape(5, K // B, B) @ H).reshape(5, K)
    scale = np.abs(deq).reshape(5, K // B, B).sum(-1, keepdims=True) / math.sqrt(B)
    bound = np.broadcast_to(scale, (5, K // B, B)).reshape(5, K) * (math.log2(B) + 2) * 2.0 ** -23
    assert np.all(np.abs(w - ref) <= bound)


def test_dequantize_inverts_rotated_quantization_within_error_bound():
    """W -> rotate + quantize -> dequantize + un-rotate: per row the L2 error
    is at most that of the rotated-basis codes, sqrt(K) * s / 2, because R is
    orthogonal; without the un-rotation it would be of the order of |W|."""
    d = workloads.rotated_layer(M=1, seed=2)
    W = d["w"][:64]
    q, s, _ = oracle.quantize_rows(W, B=128, flags=oracle.REJECT_ZERO_ROWS)
    w, st = oracle.dequantize(q, s, 128)
    assert st == 0
    err = np.linalg.norm(W.astype(np.float64) - w, axis=1)
    assert np.all(err <= math.sqrt(W.shape[1]) * s.astype(np.float64) / 2 * (1 + 1e-3))
    w_plain, _ = oracle.dequantize(q, s, 0)
    assert np.all(np.linalg.norm(W.astype(np.float64) - w_plain, axis=1) > 10 * err)


def test_dequantize_argument_checks():
    q = np.zeros((2, 48), np.int8)
    s = np.ones(2, np.float32)
    assert oracle.dequantize(q, s, 3)[1] == oracle.BIT_ARG
    assert oracle.dequantize(q, s, 32)[1] == oracle.BIT_SHAPE


# --------------------------------------------------------------------------
# The forward's bf16 route
# --------------------------------------------------------------------------

def test_round_bf16_matches_torch():
    rng = np.random.Generator(np.random.PCG64(31))
    vals = np.concatenate([
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e3),
        (rng.standard_normal(200) * 1e-39).astype(np.float32),           # subnormals
        np.array([0.0, -0.0, np.inf, -np.inf, 3.4e38, -3.4e38, 1.00390625, 1.01171875,
                  1.0 + 2.0 ** -8 + 2.0 ** -20], np.float32),             # ties and near-ties
    ])
    ref = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()
    got = np.array([oracle.round_bf16(v) for v in vals], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert math.isnan(oracle.round_bf16(float("nan")))


def test_fwd_bf16_exact_when_inputs_are_representable():
    """Small-integer x (exact in bf16), integer codes, power-of-two scales:
    every step is exact, so y is the integer product times s_w plus bias."""
    rng = np.random.Generator(np.random.PCG64(32))
    x = rng.integers(-8, 9, size=(5, 96)).astype(np.float32)
    q = rng.integers(-127, 128, size=(7, 96)).astype(np.int8)
    sw = (2.0 ** -rng.integers(0, 8, size=7)).astype(np.float32)
    b = rng.integers(-4, 5, size=7).astype(np.float32)
    y, xr, st = oracle.fwd_bf16(x, q, sw, b, 0)
    assert st == 0 and np.array_equal(xr, x)
    ref = (x.astype(np.int64) @ q.astype(np.int64).T).astype(np.float64) * sw + b
    assert np.array_equal(y, ref.astype(np.float32))


def test_fwd_bf16_equals_x_times_dequantized_weight():
    """(bf16(x R)) (s q)^T = x ((s q) R)^T = x W_hat^T up to the bf16 rounding
    of x R (2^-9 relative per element): rotating the activations stands in
    for un-rotating the weight ([CR] third commit note, item 2)."""
    d = workloads.rotated_layer(M=1, seed=3)
    x = workloads.normal((6, 5376), 1.0, 33)
    W = d["w"][:40]
    q, s, _ = oracle.quantize_rows(W, B=128, flags=oracle.REJECT_ZERO_ROWS)
    y, xr, st = oracle.fwd_bf16(x, q, s, None, 128)
    assert st == 0
    w_hat, _ = oracle.dequantize(q, s, 128)
    ref = x.astype(np.float64) @ w_hat.astype(np.float64).T
    xR, _ = oracle.hadamard_rows(x, 128)
    D = np.abs(xR.astype(np.float64)) @ np.abs(q.astype(np.float64) * s[:, None]).T
    assert np.all(np.abs(y - ref) <= D * (2.0 ** -9 + 1e-5))
    y0, _, _ = oracle.fwd_bf16(x, q, s, None, 0)     # the stored basis without rotating x
    assert np.abs(y0 - ref).max() > 100 * np.abs(y - ref).max()


# --------------------------------------------------------------------------
# Integer GEMMs
# --------------------------------------------------------------------------

def _brute(A, B, M, N, C, a_at, b_at):
    out = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            out[m][n] = sum(int(a_at(A, m, c)) * int(b_at(B, n, c)) for c in range(C))
    return np.array(out, dtype=np.int64)


def test_gemm_brute_force_tiny():
    rng = np.random.Generator(np.random.PCG64(11))
    M, N, C = 3, 5, 7
    A = rng.integers(-127, 128, size=(M, C)).astype(np.int8)
    Bt = rng.integers(-127, 128, size=(N, C)).astype(np.int8)
    out, st = oracle.gemm_nt(A, Bt)
    assert st == 0
    assert np.array_equal(out, _brute(A, Bt, M, N, C, lambda a, m, c: a[m, c], lambda b, n, c: b[n, c]))
    Bn = rng.integers(-127, 128, size=(C, N)).astype(np.int8)
    out, st = oracle.gemm_nn(A, Bn)
    assert np.array_equal(out, _brute(A, Bn, M, N, C, lambda a, m, c: a[m, c], lambda b, n, c: b[c, n]))
    At = rng.integers(-127, 128, size=(C, M)).astype(np.int8)
    out, st = oracle.gemm_tn(At, Bn)
    assert np.array_equal(out, _brute(At, Bn, M, N, C, lambda a, m, c: a[c, m], lambda b, n, c: b[c, n]))


def test_gemm_matches_numpy_int64():
    rng = np.random.Generator(np.random.PCG64(12))
    A = rng.integers(-127, 128, size=(37, 300)).astype(np.int8)
    Bt = rng.integers(-127, 128, size=(45, 300)).astype(np.int8)
    Bn = rng.integers(-127, 128, size=(300, 45)).astype(np.int8)
    At = rng.integers(-127, 128, size=(300, 37)).astype(np.int8)
    i64 = lambda a: a.astype(np.int64)
    assert np.array_equal(oracle.gemm_nt(A, Bt)[0], i64(A) @ i64(Bt).T)
    assert np.array_equal(oracle.gemm_nn(A, Bn)[0], i64(A) @ i64(Bn))
    assert np.array_equal(oracle.gemm_tn(At, Bn)[0], i64(At).T @ i64(Bn))


def test_gemm_closed_forms_and_int32_limit():
    """All-127 operands give 16129*C.  The pages' limit C = 131,071
    (mini_trainer, contraction paragraph) is floor((2^31-1) / 128^2): no int8
    dot product of that length leaves int32; at it all-127 gives 2,114,044,159."""
    limit = int(golden()["int32_contraction_limit"])
    assert limit == oracle.MAX_CONTRACTION == (2 ** 31 - 1) // (128 * 128)
    assert 128 * 128 * limit < 2 ** 31 <= 128 * 128 * (limit + 1)
    A = np.full((1, limit), 127, np.int8)
    out, st = oracle.gemm_nt(A, A)
    assert st == 0 and out[0, 0] == 16129 * limit == 2114044159
    out, st = oracle.gemm_nt(A, -A)
    assert st == 0 and out[0, 0] == -2114044159
    # beyond the limit the forward reports its contraction (in_features) as
    # unsupported; the backward products combine chunks in int64 (below)
    x = np.zeros((1, limit + 1), np.float32)
    w = np.zeros((1, limit + 1), np.int8)
    y, _, _, st = oracle.fwd(x, w, np.zeros(1, np.float32))
    assert st == oracle.BIT_UNSUPPORTED


def test_bwd_dx_beyond_int32_combines_in_int64():
    """140,000 output classes of all-127 codes sum to 16129 * 140000 =
    2,258,060,000 > 2^31 - 1: the input gradient's dot products leave int32,
    and the page combines bounded int32 chunk sums in int64 before scaling,
    which is the exact integer sum, converted to float32 once."""
    N, M, K = 140000, 2, 32
    dy = np.ones((M, N), np.float32)
    dy[1] = -1.0
    wq = np.full((N, K), 127, np.int8)
    dx, rq, s1, st = oracle.bwd_dx(dy, wq, np.ones(N, np.float32), 0)
    acc = 16129 * N
    assert acc > 2 ** 31 - 1 and st == 0
    assert np.all(rq[0] == 127) and np.all(rq[1] == -127)
    assert np.array_equal(dx[0], np.full(K, np.float32(acc) * s1[0], np.float32))
    assert np.array_equal(dx[1], np.full(K, np.float32(-acc) * s1[1], np.float32))


def test_bwd_long_contractions_match_numpy_int64():
    """dX over 150,000 output classes and dW over 140,000 tokens: the oracle's
    sums against numpy's int64 matmul of the same codes."""
    rng = np.random.Generator(np.random.PCG64(41))
    N, M, K = 150000, 3, 16
    dy = rng.standard_normal((M, N)).astype(np.float32)
    wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sw = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    dx, rq, s1, st = oracle.bwd_dx(dy, wq, sw, 0)
    assert st == 0
    acc = rq.astype(np.int64) @ wq.astype(np.int64)
    assert np.array_equal(dx, acc.astype(np.float32) * s1[:, None])
    M, N = 140000, 3
    dy = rng.standard_normal((M, N)).astype(np.float32)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-2, M).astype(np.float32)
    dw, db, rqc, s2, st = oracle.bwd_dw(dy, xq, sx)
    assert st == 0
    acc = rqc.astype(np.int64).T @ xq.astype(np.int64)
    assert np.array_equal(dw, acc.astype(np.float32) * s2[:, None])


# --------------------------------------------------------------------------
# Layer forward and backward
# --------------------------------------------------------------------------

def test_fwd_exact_when_inputs_are_representable():
    """x = s_x q_x and W = s_w q_w with power-of-two scales: the layer output
    equals the float64 product up to the float32 epilogue rounding."""
    rng = np.random.Generator(np.random.PCG64(13))
    M, K, N = 17, 96, 40
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8); qx[:, 0] = 127
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sx = (2.0 ** -rng.integers(0, 8, size=M)).astype(np.float32)
    sw = (2.0 ** -rng.integers(4, 10, size=N)).astype(np.float32)
    b = workloads.normal((N,), 0.01, 14)
    x = qx.astype(np.float32) * sx[:, None]
    y, xq, sxo, st = oracle.fwd(x, qw, sw, b)
    assert st == 0 and np.array_equal(xq, qx) and np.array_equal(sxo, sx)
    ref = (x.astype(np.float64) @ (qw.astype(np.float64) * sw[:, None]).T) + b
    assert np.abs(y - ref).max() <= 1e-6 * np.abs(ref).max()


def _prep_weight(w, B):
    q, s, st = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
    assert st == 0
    return q, s


def test_fwd_rotation_reduces_error_with_outliers():
    """The int8 route approximates x W^T + b; with outlier channels the
    rotated route (both operands rotated) is closer than the plain one
    (OneTrainer PR #1681: the benefit tracks the outlier ratio)."""
    d = workloads.tiny_layer()
    x, w, b = d["x"], d["w"], d["bias"]
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    errs = {}
    for B in (0, 256):
        wq, sw = _prep_weight(w, B)
        y, _, _, st = oracle.fwd(x, wq, sw, b, B)
        assert st == 0
        errs[B] = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert errs[256] < 0.5 * errs[0]
    assert errs[256] < 0.03


def test_bwd_dx_exact_case():
    """s_w = 1 and integer dY rows containing +-127: dYq_r = dY, s' = 1, so dX
    is the integer product dY W_q (numpy int64)."""
    rng = np.random.Generator(np.random.PCG64(15))
    M, N, K = 9, 48, 80
    dyi = rng.integers(-127, 128, size=(M, N)); dyi[:, 3] = 127
    wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    dx, q, s1, st = oracle.bwd_dx(dyi.astype(np.float32), wq, np.ones(N, np.float32))
    assert st == 0 and np.array_equal(q, dyi) and np.all(s1 == 1)
    assert np.array_equal(dx, (dyi @ wq.astype(np.int64)).astype(np.float32))


def test_bwd_dx_rotated_returns_to_input_basis():
    """For a rotated layer dL/dx = (dY W_rot) R^T = dY W: the oracle's dX
    approximates dY W in the original basis and not dY W_rot."""
    d = workloads.tiny_layer()
    w, dy = d["w"], d["dy"]
    wq, sw = _prep_weight(w, 256)
    dx, _, _, st = oracle.bwd_dx(dy, wq, sw, 256)
    assert st == 0
    ref = dy.astype(np.float64) @ w.astype(np.float64)
    rot = dy.astype(np.float64) @ (wq.astype(np.float64) * sw[:, None])
    assert np.linalg.norm(dx - ref) / np.linalg.norm(ref) < 0.03
    assert np.linalg.norm(dx - rot) / np.linalg.norm(rot) > 0.5


def test_bwd_dw_exact_case_and_bias_grad():
    """s_x = 1 and integer dY columns containing +-127: dYq_c = dY, s'' = 1,
    dW = dY^T X_q (numpy int64); db = column sums of dY."""
    rng = np.random.Generator(np.random.PCG64(16))
    M, N, K = 23, 40, 64
    dyi = rng.integers(-127, 128, size=(M, N)); dyi[4, :] = -127
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    dw, db, q, s2, st = oracle.bwd_dw(dyi.astype(np.float32), xq, np.ones(M, np.float32))
    assert st == 0 and np.array_equal(q, dyi) and np.all(s2 == 1)
    assert np.array_equal(dw, (dyi.T @ xq.astype(np.int64)).astype(np.float32))
    assert np.array_equal(db, dyi.sum(0).astype(np.float32))


def test_bwd_dw_approximates_float_gradient():
    d = workloads.tiny_layer()
    xq, sx, _ = oracle.quantize_rows(d["x"], B=256)
    dy = d["dy"]
    dw, db, _, _, st = oracle.bwd_dw(dy, xq, sx)
    assert st == 0
    ref = dy.astype(np.float64).T @ (xq.astype(np.float64) * sx[:, None])
    assert np.linalg.norm(dw - ref) / np.linalg.norm(ref) < 0.03
    assert np.allclose(db, dy.astype(np.float64).sum(0), rtol=1e-6, atol=1e-6)


def test_bwd_zero_columns_are_legal():
    dy = workloads.normal((8, 32), 1.0, 17)
    dy[:, 5] = 0.0
    q, s2, db, st = oracle.bwd_prep_cols(dy, np.ones(8, np.float32))
    assert st == 0 and s2[5] == 0 and not q[:, 5].any() and db[5] == 0


# --------------------------------------------------------------------------
# Philox4x32-10 and stochastic rounding
# --------------------------------------------------------------------------

CURAND = "/usr/local/cuda/lib64/libcurand.so"


def _curand_host_philox(seed: int, n: int) -> np.ndarray:
    lib = ctypes.CDLL(CURAND)
    g = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(g), 161) == 0  # PHILOX4_32_10
    assert lib.curandSetPseudoRandomGeneratorSeed(g, ctypes.c_ulonglong(seed)) == 0
    out = np.zeros(n, dtype=np.uint32)
    assert lib.curandGenerate(g, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
    lib.curandDestroyGenerator(g)
    return out


@pytest.mark.skipif(not os.path.exists(CURAND), reason="cuRAND host library not present")
def test_philox_matches_curand_host_generator():
    """cuRAND's host Philox4x32-10 (seed = key) emits block j from counter
    (j / 65536, 0, j % 65536, 0); the oracle must reproduce every word."""
    rng = np.random.Generator(np.random.PCG64(18))
    for seed in (0, 7, 0x123456789ABCDEF0):
        out = _curand_host_philox(seed, 4 * 65536 * 2)
        key = [seed & 0xFFFFFFFF, seed >> 32]
        blocks = list(range(0, 40)) + list(rng.integers(0, 2 * 65536, size=300))
        for j in blocks:
            j = int(j)
            ctr = [j // 65536, 0, j % 65536, 0]
            assert np.array_equal(oracle.philox4x32_10(ctr, key), out[4 * j:4 * j + 4]), (seed, j)
        # the stochastic-rounding uniform: element e at step z uses counter
        # (e >> 2, 0, z, 0) and word e & 3, top 24 bits
        for j in blocks[:64]:
            j = int(j)
            x, z = j // 65536, j % 65536
            for w in range(4):
                assert oracle.sr_u24(seed, z, 4 * x + w) == int(out[4 * j + w]) >> 8


def test_u24_is_uniform():
    """Chi-square over 256 bins of u24 >> 16 for 2^17 consecutive elements."""
    n = 1 << 17
    u = np.array([oracle.sr_u24(1234, 3, e) for e in range(n)], np.int64)
    assert u.min() >= 0 and u.max() < (1 << 24)
    counts = np.bincount(u >> 16, minlength=256)
    exp = n / 256
    chi2 = ((counts - exp) ** 2 / exp).sum()
    # 255 degrees of freedom: mean 255, sd ~22.6; 6 sd bound
    assert chi2 < 255 + 6 * 22.6


@pytest.mark.parametrize("v", [0.25, -0.25, 3.7, -3.7, 126.9, -126.9, 0.0,
                               5.0, -101.0, 1.0 / 3.0, 2.0 ** -25, -(2.0 ** -23)])
def test_sr_expectation_by_enumeration(v):
    """Over all 2^24 uniforms, E[q] = floor(v) + ceil(frac * 2^24) / 2^24, so
    |E[q] - v| < 2^-24: stochastic rounding is unbiased to 24 bits."""
    v32 = float(np.float32(v))
    E = oracle.sr_expectation_enum(v32)
    f = math.floor(v32)
    frac = v32 - f
    assert E == f + math.ceil(frac * 2 ** 24) / 2 ** 24
    assert abs(E - v32) < 2.0 ** -24
    if v32 == f:
        assert E == v32


def test_sr_identity_when_values_are_codes():
    """SGD with lr = 0 on a row with a power-of-two scale leaves every code
    an integer after scaling, so the stochastic requant is exact."""
    rng = np.random.Generator(np.random.PCG64(19))
    q = rng.integers(-127, 128, size=(6, 64)).astype(np.int8); q[:, 0] = -127
    s = (2.0 ** -rng.integers(3, 9, size=6)).astype(np.float32)
    g = workloads.normal((6, 64), 1.0, 20)
    q2, s2, *_, st = oracle.update_sr(q, s, g, oracle.SGD, 0.0, seed=5, step=1)
    assert st == 0 and np.array_equal(q2, q) and np.array_equal(s2, s)


def test_sr_unbiased_over_seeds():
    """The mean of the requantized weight over many seeds approaches the
    float update (5 sigma)."""
    d = workloads.update_state(4, 64, seed=2)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    w1, *_ = oracle.update_float(q, s, d["grad"], oracle.SGD, 0.05, step=1)
    n = 400
    acc = np.zeros_like(w1, np.float64)
    for seed in range(n):
        q2, s2, *_ = oracle.update_sr(q, s, d["grad"], oracle.SGD, 0.05, seed=seed, step=1)
        acc += q2.astype(np.float64) * s2[:, None]
    mean = acc / n
    step = (np.abs(w1).max(1) / 127.0)[:, None]
    sigma = 0.5 * step / math.sqrt(n)
    assert np.all(np.abs(mean - w1) <= 5 * sigma + 1e-9)


# --------------------------------------------------------------------------
# Optimizer steps against torch.optim / torch autograd (float64)
# --------------------------------------------------------------------------

def _f32(v: float) -> float:
    """The float32 value the C ABI receives for a hyper-parameter."""
    return float(np.float32(v))


def _dequant(q, s):
    return q.astype(np.float64) * s.astype(np.float64)[:, None]


def test_sgd_step_matches_torch():
    d = workloads.update_state(8, 96, seed=3)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    w, *_, st = oracle.update_float(q, s, d["grad"], oracle.SGD, 1e-2, step=1)
    assert st == 0
    p = torch.nn.Parameter(torch.from_numpy(q.astype(np.float32) * s[:, None]).double())
    opt = torch.optim.SGD([p], lr=_f32(1e-2))
    p.grad = torch.from_numpy(d["grad"]).double()
    opt.step()
    assert np.abs(w - p.detach().numpy()).max() <= 1e-8


@pytest.mark.parametrize("warm", [False, True])
def test_adamw_step_matches_torch(warm):
    d = workloads.update_state(8, 96, seed=4, warm=warm)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    lr, wd, t = 1e-3, 0.01, d["step"]
    w, m, v, *_, st = oracle.update_float(q, s, d["grad"], oracle.ADAMW, lr, step=t,
                                          m=d["m"], v=d["v"], wd=wd)
    assert st == 0
    p = torch.nn.Parameter(torch.from_numpy(q.astype(np.float32) * s[:, None]).double())
    opt = torch.optim.AdamW([p], lr=_f32(lr), betas=(_f32(0.9), _f32(0.999)), eps=_f32(1e-8),
                            weight_decay=_f32(wd))
    p.grad = torch.from_numpy(d["grad"]).double()
    opt.state[p] = {"step": torch.tensor(float(t - 1)),
                    "exp_avg": torch.from_numpy(d["m"]).double(),
                    "exp_avg_sq": torch.from_numpy(d["v"]).double()}
    opt.step()
    st_t = opt.state[p]
    assert np.allclose(m, st_t["exp_avg"].numpy(), rtol=1e-5, atol=1e-12)
    assert np.allclose(v, st_t["exp_avg_sq"].numpy(), rtol=1e-5, atol=1e-16)
    assert np.abs(w - p.detach().numpy()).max() <= 1e-6 * np.abs(w).max()


def test_adamw_first_step_closed_form():
    """At step 1 from zero moments the bias corrections cancel: m_hat = g and
    v_hat = g^2, so w' = w (1 - lr wd) - lr g / (|g| + eps), independent of
    the betas.  A dropped correction, swapped betas or a wrong sign move it
    by orders of magnitude more than float32 rounding."""
    d = workloads.update_state(8, 96, seed=8)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    lr, wd, eps = 1e-3, 0.01, 1e-8
    w, m, v, *_, st = oracle.update_float(q, s, d["grad"], oracle.ADAMW, lr, step=1,
                                          m=d["m"], v=d["v"], wd=wd)
    assert st == 0
    w0 = _dequant(q, s)
    g = d["grad"].astype(np.float64)
    want = w0 * (1.0 - lr * wd) - lr * g / (np.abs(g) + eps)
    assert np.abs(w - want).max() <= 1e-6 * (np.abs(w0).max() + lr)
    assert np.allclose(m, 0.1 * g, rtol=1e-6) and np.allclose(v, 0.001 * g * g, rtol=1e-5)


def test_adamw_zero_gradient_is_pure_decoupled_decay():
    """With g = 0 and zero moments the Adam term vanishes and only the
    decoupled decay remains: w' = w (1 - lr wd).  Weight decay folded into
    the gradient (L2) would instead move every weight by about lr."""
    d = workloads.update_state(4, 64, seed=9)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    lr, wd = 1e-3, 0.01
    zero = np.zeros_like(d["grad"])
    w, m, v, *_, st = oracle.update_float(q, s, zero, oracle.ADAMW, lr, step=1,
                                          m=d["m"], v=d["v"], wd=wd)
    assert st == 0 and not m.any() and not v.any()
    w0 = _dequant(q, s)
    assert np.abs(w - w0 * (1.0 - lr * wd)).max() <= 1e-7 * np.abs(w0).max()


def test_weight_norm_step_matches_torch_autograd():
    """Row-wise weight norm (dim=0): w = g * v / ||v||.  torch autograd gives
    dL/dg and dL/dv for dL/dw = grad; torch AdamW then steps g and v."""
    d = workloads.update_state(6, 128, seed=5, weight_norm=True)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    lr, wd = 1e-3, 0.01
    wv, m, v, g, gm, gv, st = oracle.update_float(
        q, s, d["grad"], oracle.ADAMW, lr, step=1, m=d["m"], v=d["v"], wd=wd,
        g=d["g"], g_m=d["g_m"], g_v=d["g_v"])
    assert st == 0
    vp = torch.nn.Parameter(torch.from_numpy(_dequant(q, s)))
    gp = torch.nn.Parameter(torch.from_numpy(d["g"].astype(np.float64)))
    w_eff = gp[:, None] * vp / vp.norm(dim=1, keepdim=True)
    (w_eff * torch.from_numpy(d["grad"]).double()).sum().backward()
    # direction gradient is orthogonal to the direction
    assert (vp.grad * vp.detach()).sum(1).abs().max().item() <= 1e-12
    opt = torch.optim.AdamW([vp, gp], lr=_f32(lr), betas=(_f32(0.9), _f32(0.999)),
                            eps=_f32(1e-8), weight_decay=_f32(wd))
    opt.step()
    assert np.abs(wv - vp.detach().numpy()).max() <= 1e-6 * np.abs(wv).max()
    assert np.allclose(g, gp.detach().numpy(), rtol=1e-6)
    assert np.allclose(m, opt.state[vp]["exp_avg"].numpy(), rtol=1e-4, atol=1e-12)
    assert np.allclose(gm, opt.state[gp]["exp_avg"].numpy(), rtol=1e-4, atol=1e-12)


def test_weight_norm_effective_rows_have_norm_g():
    d = workloads.update_state(5, 64, seed=6, weight_norm=True)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    q2, s2, m, v, g2, gm, gv, st = oracle.update_sr(
        q, s, d["grad"], oracle.ADAMW, 1e-3, seed=1, step=1, m=d["m"], v=d["v"],
        g=d["g"], g_m=d["g_m"], g_v=d["g_v"])
    assert st == 0
    w_eff = g2[:, None] * q2.astype(np.float64) / np.linalg.norm(q2.astype(np.float64), axis=1)[:, None]
    assert np.allclose(np.linalg.norm(w_eff, axis=1), g2, rtol=1e-12)


def test_weight_norm_rejects_zero_direction():
    d = workloads.update_state(3, 32, seed=7, weight_norm=True)
    q, s, _ = oracle.quantize_rows(d["w"])
    q[1] = 0
    s[1] = 0
    q2, s2, m, v, g2, *_, st = oracle.update_sr(
        q, s, d["grad"], oracle.ADAMW, 1e-3, seed=1, step=1, m=d["m"], v=d["v"],
        g=d["g"], g_m=d["g_m"], g_v=d["g_v"])
    assert st == oracle.BIT_ZERO_ROW
    assert not q2[1].any() and g2[1] == d["g"][1] and not m[1].any()
    assert q2[0].any() and q2[2].any()


def test_update_argument_checks():
    q = np.ones((2, 16), np.int8)
    s = np.ones(2, np.float32)
    g = np.zeros((2, 16), np.float32)
    assert oracle.update_sr(q, s, g, oracle.SGD, 0.1, seed=0, step=0)[-1] == oracle.BIT_ARG
    assert oracle.update_sr(q, s, g, oracle.SGD, 0.1, seed=0, step=1, wd=0.1)[-1] == oracle.BIT_ARG
    assert oracle.update_sr(q, s, g, 7, 0.1, seed=0, step=1)[-1] == oracle.BIT_ARG


# ---------------------------------------------------------------- SwiGLU gate
U32 = 2.0 ** -24  # unit roundoff of float32


def test_exp_within_one_ulp_of_float64():
    """The oracle's exp (Cody-Waite reduction + Taylor series) against numpy's
    float64 exp on a dense sweep: under 1 ulp of float32 where the result is
    a normal number, under one subnormal step below that; exact at 0."""
    xs = np.concatenate([np.linspace(-110, 95, 100001, dtype=np.float32),
                         np.float32([0.0, -0.0, 1e-30, -1e-30, 1e-7, 88.72, -87.3, -103.9])])
    e = oracle.exp_array(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    normal = (ref > 1.1754944e-38) & (ref < 3.4028235e38)
    ulp = np.spacing(ref[normal].astype(np.float32)).astype(np.float64)
    assert (np.abs(e[normal] - ref[normal]) / ulp).max() < 1.0
    low = ref <= 1.1754944e-38
    assert np.abs(e[low] - ref[low]).max() <= 2.0 ** -149
    assert oracle.exp(0.0) == 1.0
    assert oracle.exp(89.0) == math.inf and oracle.exp(math.inf) == math.inf
    assert oracle.exp(-110.0) == 0.0 and oracle.exp(-math.inf) == 0.0
    assert math.isnan(oracle.exp(math.nan))
    # e^x at the float32 nearest k ln 2: 2^k e^(x - k ln 2) to the same bound
    for k in range(-120, 120, 7):
        x = float(np.float32(k * math.log(2.0)))
        ref = 2.0 ** k * math.exp(x - k * math.log(2.0))
        assert abs(oracle.exp(x) - ref) < float(np.spacing(np.float32(ref)))


def _silu64(a):
    return a / (1.0 + np.exp(-a))


def _swiglu_inputs(M, F, seed):
    ab = workloads.normal((M, 2 * F), 1.28, seed)
    ab[0, :4] = np.float32([0.0, -0.0, 100.0, -100.0])   # silu = 0, 0, a, -0
    ab[1, :3] = np.float32([-120.0, 90.0, 1e-30])
    return ab


def test_swiglu_h_against_float64():
    """h = silu(a) * b within 4 float32 roundings of the float64 value: the
    exp (< 1 ulp), 1 + e, the division and the product.  Below a = -88.7,
    e^-a overflows float32 and silu(a) = a/inf = -0, where the true value
    |a| e^a is under 3e-37: an absolute allowance of that size."""
    M, F = 64, 512
    ab = _swiglu_inputs(M, F, 11)
    h = oracle.swiglu_h(ab).astype(np.float64)
    a, b = ab[:, :F].astype(np.float64), ab[:, F:].astype(np.float64)
    ref = _silu64(a) * b
    tiny = 3e-37 * np.abs(b)
    assert np.all(np.abs(h - ref) <= 4 * U32 * np.abs(ref) + tiny)
    assert h[0, 0] == 0.0 and h[0, 2] == np.float32(100.0) * ab[0, F + 2]
    assert h[0, 3] == 0.0 and np.signbit(h[0, 3]) != np.signbit(ab[0, F + 3])
    # torch's own silu agrees to the same bound
    t = torch.nn.functional.silu(torch.from_numpy(a)).numpy() * b
    assert np.all(np.abs(h - t) <= 4 * U32 * np.abs(t) + tiny)


def test_swiglu_quantize_is_the_row_quantization_of_h():
    """The second projection's saved input: per-row quantization (pinned
    above) of h, with zero rows and the non-finite flag carried through."""
    M, F = 48, 384
    ab = _swiglu_inputs(M, F, 12)
    ab[5, :F] = 0.0            # a = 0: h row is zero
    q, s, st = oracle.swiglu_quantize(ab)
    rq, rs, rst = oracle.quantize_rows(oracle.swiglu_h(ab), B=0)
    assert st == rst == 0 and s[5] == 0 and not q[5].any()
    assert np.array_equal(q, rq) and np.array_equal(s, rs)
    # every code reconstructs h within half a step
    h = oracle.swiglu_h(ab).astype(np.float64)
    assert np.all(np.abs(q * s[:, None].astype(np.float64) - h) <= s[:, None] / 2 * (1 + 1e-6))
    ab[7, F + 3] = np.nan
    assert oracle.swiglu_quantize(ab)[2] == oracle.BIT_NONFINITE


def test_swiglu_bwd_against_torch_autograd():
    """[da | db] against torch autograd of silu(a) * b in float64, within a
    few float32 roundings of each term's magnitude."""
    M, F = 40, 256
    ab = _swiglu_inputs(M, F, 13)
    dh = workloads.normal((M, F), 1.0, 14)
    dab = oracle.swiglu_bwd(ab, dh).astype(np.float64)
    a = torch.from_numpy(ab[:, :F].astype(np.float64)).requires_grad_()
    b = torch.from_numpy(ab[:, F:].astype(np.float64)).requires_grad_()
    (torch.nn.functional.silu(a) * b).backward(torch.from_numpy(dh.astype(np.float64)))
    a64, b64, g = a.detach().numpy(), b.detach().numpy(), dh.astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-a64))
    mag_a = np.abs(g * b64) * (sig + np.abs(a64) * sig * (1 - sig))
    tiny = 1e-35 * np.abs(g) * (1 + np.abs(b64))  # e^-a overflow below a = -88.7
    assert np.all(np.abs(dab[:, :F] - a.grad.numpy()) <= 10 * U32 * mag_a + tiny)
    mag_b = np.abs(g * _silu64(a64))
    assert np.all(np.abs(dab[:, F:] - b.grad.numpy()) <= 6 * U32 * mag_b + tiny)


def test_fwd_quantized_is_the_forward_after_its_quantization():
    """The forward from codes equals the whole forward when given the codes
    and scales that the forward's own quantization produces (bit for bit),
    and is the exact product for unit scales."""
    x = workloads.normal((37, 256), 1.0, 31)
    w = workloads.normal((48, 256), 0.02, 32)
    b = workloads.normal((48,), 0.01, 33)
    wq, sw, _ = oracle.quantize_rows(w, flags=oracle.REJECT_ZERO_ROWS)
    y, xq, sx, st = oracle.fwd(x, wq, sw, b, 0)
    y2, st2 = oracle.fwd_quantized(xq, sx, wq, sw, b)
    assert st == st2 == 0 and np.array_equal(y, y2)
    rng = np.random.Generator(np.random.PCG64(34))
    xi = rng.integers(-127, 128, (5, 64)).astype(np.int8)
    wi = rng.integers(-127, 128, (16, 64)).astype(np.int8)
    y3, _ = oracle.fwd_quantized(xi, np.ones(5, np.float32), wi, np.ones(16, np.float32))
    assert np.array_equal(y3, (xi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float32))


# ---------------------------------------------------------------- MuonAuxAdamW
NS_COEF = (3.4445, -4.7750, 2.0315)


def _ns5_by_svd(U, steps=5):
    """The quintic Newton-Schulz map acts on singular values only: the same
    O from numpy's SVD and the scalar iteration s -> a s + b s^3 + c s^5."""
    a, b, c = NS_COEF
    U64 = U.astype(np.float64)
    u, sv, vt = np.linalg.svd(U64, full_matrices=False)
    x = sv / (np.linalg.norm(U64) + 1e-7)
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return (u * x) @ vt


@pytest.mark.parametrize("R,C", [(48, 80), (80, 48), (64, 64), (1, 32)])
def test_newton_schulz_matches_the_svd_closed_form(R, C):
    U = workloads.normal((R, C), 1e-3, R * 7 + C)
    O = oracle.newton_schulz5(U)
    ref = _ns5_by_svd(U)
    assert np.abs(O - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    # after five steps every singular value sits in the iteration's band
    sv = np.linalg.svd(O, compute_uv=False)
    assert sv.min() > 0.6 and sv.max() < 1.25


def test_newton_schulz_zero_and_one_step():
    assert not oracle.newton_schulz5(np.zeros((8, 16), np.float32)).any()
    U = workloads.normal((16, 24), 1.0, 3)
    O1 = oracle.newton_schulz5(U, steps=1)
    assert np.abs(O1 - _ns5_by_svd(U, steps=1)).max() <= 1e-12


def test_muon_momentum_against_torch_lerp():
    """M' and the Nesterov blend against torch's lerp form in float64 (the
    published implementation's momentum.lerp_(g, 1-beta); g.lerp_(m, beta)),
    within float32 roundings of each term."""
    G = workloads.normal((64, 96), 1e-3, 4)
    M = workloads.normal((64, 96), 1e-3, 5)
    M2, U = oracle.muon_momentum(G, M, 0.95)
    g, m = torch.from_numpy(G.astype(np.float64)), torch.from_numpy(M.astype(np.float64))
    m.lerp_(g, 1 - 0.95)
    u = g.clone().lerp_(m, 0.95)
    mag = np.abs(G.astype(np.float64)) + np.abs(M.astype(np.float64))
    assert np.all(np.abs(M2 - m.numpy()) <= 4 * 2.0 ** -24 * mag)
    assert np.all(np.abs(U - u.numpy()) <= 8 * 2.0 ** -24 * mag)
    # beta = 0: plain gradient, exactly
    M3, U3 = oracle.muon_momentum(G, M, 0.0)
    assert np.array_equal(M3, G) and np.array_equal(U3, G)


def test_muon_update_step_and_requant():
    """The float step w*(1-lr*wd) - lr*max(1,N/K)^0.5*O against torch's
    mul_/add_ in float64; a zero update with no decay leaves every code and
    scale unchanged; the stochastic rounding is that of the other updates."""
    N, K = 96, 64   # N > K: the step size is scaled by sqrt(N/K)
    w = workloads.normal((N, K), 0.02, 6)
    q, s, _ = oracle.quantize_rows(w, flags=oracle.REJECT_ZERO_ROWS)
    O = workloads.normal((N, K), 0.1, 7)
    lr, wd = 0.02, 0.01
    q2, s2, st = oracle.update_muon_sr(q, s, O, lr, wd, seed=9, step=3)
    assert st == 0
    p = torch.from_numpy(q.astype(np.float64) * s[:, None].astype(np.float64))
    p.mul_(1 - lr * wd).add_(torch.from_numpy(O.astype(np.float64)), alpha=-lr * math.sqrt(N / K))
    ref = p.numpy()
    # dequantized new codes within one code step of the torch value per row
    deq = q2.astype(np.float64) * s2[:, None].astype(np.float64)
    assert np.all(np.abs(deq - ref) <= s2[:, None] * (1 + 1e-5))
    q3, s3, st = oracle.update_muon_sr(q, s, np.zeros_like(O), lr, 0.0, seed=9, step=3)
    assert st == 0 and np.array_equal(q3, q) and np.array_equal(s3, s)


def test_adamw_vector_matches_torch():
    n = 300
    p0 = workloads.normal((n,), 0.01, 8)
    g = workloads.normal((n,), 1e-3, 9)
    m = workloads.normal((n,), 1e-4, 10)
    v = np.square(workloads.normal((n,), 1e-3, 11))
    p1, m1, v1, st = oracle.adamw_vector(p0, g, m, v, 1e-3, step=10, wd=0.01)
    assert st == 0
    t = torch.from_numpy(p0.astype(np.float64)).requires_grad_()
    opt = torch.optim.AdamW([t], lr=float(np.float32(1e-3)), weight_decay=float(np.float32(0.01)),
                            betas=(float(np.float32(0.9)), float(np.float32(0.999))),
                            eps=float(np.float32(1e-8)))
    opt.state[t]["step"] = torch.tensor(9.0, dtype=torch.float64)
    opt.state[t]["exp_avg"] = torch.from_numpy(m.astype(np.float64))
    opt.state[t]["exp_avg_sq"] = torch.from_numpy(v.astype(np.float64))
    t.grad = torch.from_numpy(g.astype(np.float64))
    opt.step()
    assert np.all(np.abs(p1 - t.detach().numpy()) <= 1e-6 * (np.abs(p0) + 1e-3))
