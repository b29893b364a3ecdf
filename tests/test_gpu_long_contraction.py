"""GPU parity of the backward products whose contraction is longer than the
int32-safe 131,071 (mini_trainer quantized-training doc, contraction
paragraph): the input gradient over N output classes and the weight gradient
over M tokens run in splits whose int32 partial sums are combined in int64
before scaling.  The integer sums are exact and every float step follows the
oracle's order, so dX and dW are compared bit for bit (db, a float64 sum in
another order, within the float bound)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import assert_close, dev, host, new_status, status_word

pytestmark = pytest.mark.gpu

LIMIT = ql.QL_MAX_CONTRACTION


def _ws(M, N, K, B, combined=False):
    n = (ql.qlinear_bwd_workspace_bytes if combined else ql.qlinear_workspace_bytes)(M, N, K, B)
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def _dx(dy_t, wq, sw, B, dxt):
    M, N = dy_t.shape
    K = wq.shape[1]
    dx = torch.empty((M, K), dtype=dxt, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dx(dy_t, wq, sw, B, dx, _ws(M, N, K, B), st)
    assert status_word(st) == 0
    return dx


def _as_dtype(ref, dt):
    return torch.from_numpy(ref).to(dt).float().numpy()


@pytest.mark.parametrize("M,N,K,B,dyt,dxt", [
    (40, 140000, 256, 0, torch.float32, torch.float32),       # 2 splits, single-CTA tiles
    (40, 140000, 256, 128, torch.bfloat16, torch.bfloat16),   # rotated: float32 product, then R
    (300, LIMIT + 1, 128, 0, torch.bfloat16, torch.float32),  # first N past the limit, CTA pairs
    (17, 400000, 64, 16, torch.float32, torch.float32),       # 4 splits
])
def test_dx_long_contraction_matches_oracle(M, N, K, B, dyt, dxt):
    dy = workloads.normal((M, N), 1.0, N + M)
    dy_t = torch.from_numpy(dy).to(dyt)
    w = workloads.normal((N, K), 0.02, N + 1)
    wq_np, sw_np, _ = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
    dx = _dx(dev(dy_t), dev(wq_np), dev(sw_np), B, dxt)
    rdx, _, _, st = oracle.bwd_dx(dy_t.float().numpy(), wq_np, sw_np, B)
    assert st == 0
    assert np.array_equal(host(dx), _as_dtype(rdx, dxt))


def test_dx_sums_beyond_int32_are_exact():
    """All-127 codes over 140,000 classes: each dot product is 16129 * 140000
    = 2,258,060,000, past int32; split and combined in int64 it is exact."""
    M, N, K = 3, 140000, 64
    dy = np.ones((M, N), np.float32)
    dy[1] = -1.0
    wq_np = np.full((N, K), 127, np.int8)
    sw_np = np.ones(N, np.float32)
    dx = _dx(dev(dy), dev(wq_np), dev(sw_np), 0, torch.float32)
    rdx, _, s1, _ = oracle.bwd_dx(dy, wq_np, sw_np, 0)
    assert np.array_equal(host(dx), rdx)
    assert np.all(host(dx)[0] == np.float32(16129 * N) * s1[0])


@pytest.mark.parametrize("M,N,K", [(140000, 48, 128), (LIMIT + 17, 16, 256)])
def test_dw_long_contraction_matches_oracle(M, N, K):
    x = workloads.normal((M, K), 1.0, M + 5)
    xq_np, sx_np, _ = oracle.quantize_rows(x)
    dy = workloads.normal((M, N), 1.0, M + 6)
    dy_t = torch.from_numpy(dy).to(torch.bfloat16)
    dw = torch.empty((N, K), device="cuda")
    db = torch.empty(N, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dw(dev(dy_t), dev(xq_np), dev(sx_np), dw, db, _ws(M, N, K, 0), st)
    assert status_word(st) == 0
    rdw, rdb, _, _, rst = oracle.bwd_dw(dy_t.float().numpy(), xq_np, sx_np)
    assert rst == 0
    assert np.array_equal(host(dw), rdw)
    # db: a float64 sum whose order differs (per-block partials), rounded once
    assert_close(host(db), rdb, np.abs(dy_t.float().numpy().astype(np.float64)).sum(0), what="db")


def test_combined_backward_with_long_contractions_equals_separate_calls():
    """qlinear_bwd with the dX contraction past the limit (and, in the second
    case, the dW one): bit-equal to the two separate calls."""
    for (M, N, K, B) in ((40, 140000, 256, 128), (140000, 32, 128, 0)):
        dy_t = dev(torch.from_numpy(workloads.normal((M, N), 1.0, 7)).to(torch.bfloat16))
        w = workloads.normal((N, K), 0.02, 8)
        wq_np, sw_np, _ = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
        xq_np, sx_np, _ = oracle.quantize_rows(workloads.normal((M, K), 1.0, 9), B=B)
        wq, sw, xq, sx = dev(wq_np), dev(sw_np), dev(xq_np), dev(sx_np)
        dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        dw = torch.empty((N, K), device="cuda")
        db = torch.empty(N, device="cuda")
        st = new_status()
        ql.qlinear_bwd(dy_t, wq, sw, xq, sx, B, dx, dw, db, _ws(M, N, K, B, combined=True), st)
        assert status_word(st) == 0
        dx1 = _dx(dy_t, wq, sw, B, torch.bfloat16)
        dw1 = torch.empty_like(dw)
        db1 = torch.empty_like(db)
        ql.qlinear_bwd_dw(dy_t, xq, sx, dw1, db1, _ws(M, N, K, B), st)
        assert status_word(st) == 0
        assert torch.equal(dx, dx1) and torch.equal(dw, dw1) and torch.equal(db, db1)


@pytest.mark.parametrize("M,N,K,B", [(1, 7168, 5376, 128), (17, 7168, 5376, 0), (128, 2048, 1024, 16)])
def test_dx_small_output_splits_match_oracle(M, N, K, B):
    """Outputs of at most 128 rows run as contraction splits (int32 partials
    combined in int64) to spread over the SMs: still exact."""
    dy = workloads.normal((M, N), 1.0, M + N + 3)
    w = workloads.normal((N, K), 0.02, N + 4)
    wq_np, sw_np, _ = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
    dx = _dx(dev(dy), dev(wq_np), dev(sw_np), B, torch.float32)
    rdx, _, _, st = oracle.bwd_dx(dy, wq_np, sw_np, B)
    assert st == 0 and np.array_equal(host(dx), rdx)


@pytest.mark.parametrize("M,N,K", [(4096, 64, 512), (12000, 128, 256)])
def test_dw_small_output_splits_match_oracle(M, N, K):
    x = workloads.normal((M, K), 1.0, M + 9)
    xq_np, sx_np, _ = oracle.quantize_rows(x)
    dy = workloads.normal((M, N), 1.0, M + 10)
    dw = torch.empty((N, K), device="cuda")
    st = new_status()
    ql.qlinear_bwd_dw(dev(dy), dev(xq_np), dev(sx_np), dw, None, _ws(M, N, K, 0), st)
    assert status_word(st) == 0
    rdw, _, _, _, rst = oracle.bwd_dw(dy, xq_np, sx_np)
    assert rst == 0 and np.array_equal(host(dw), rdw)
