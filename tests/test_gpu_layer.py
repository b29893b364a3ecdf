"""GPU parity of the layer's forward, input-gradient and weight-gradient calls
(tcgen05 int8 GEMMs with their epilogues) against the oracle, through the
C ABI.  Saved int8 inputs, scales and gradient codes are compared bit for
bit; float outputs within the 1e-3 relative bound (plus half a bf16 ulp for
bf16 outputs).  Integer accumulators are checked exactly by running the
GEMMs with unit scales.  Shapes span several 128x256 tiles with ragged
tails, the edge row counts 1, 15, 16, 17, and the full 2048- and
12000-token layer (sampled rows) in the configuration the benchmark times."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import (assert_close, dev, host, new_status, rotated_magnitude,
                         status_word)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ helpers
def prep_weight(w: np.ndarray, B: int):
    """Weight preparation through the library (bit-exact with the oracle,
    which test_gpu_rowops checks); returns device codes/scales."""
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_quantize_rows(dev(w), wq, sw, st, hadamard_block=B, flags=ql.QL_REJECT_ZERO_ROWS)
    assert status_word(st) == 0
    return wq, sw


def gpu_fwd(x_t, wq, sw, bias, B, yt):
    M, K = x_t.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=yt, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_fwd(x_t, wq, sw, bias, B, y, xq, sx, st)
    assert status_word(st) == 0
    return y, xq, sx


def gpu_dx(dy_t, wq, sw, B, dxt):
    M, N = dy_t.shape
    K = wq.shape[1]
    ws = torch.empty(ql.qlinear_workspace_bytes(M, N, K, B), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=dxt, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dx(dy_t, wq, sw, B, dx, ws, st)
    assert status_word(st) == 0
    return dx, ws


def gpu_dw(dy_t, xq, sx, with_db=True):
    M, N = dy_t.shape
    K = xq.shape[1]
    ws = torch.empty(ql.qlinear_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda") if with_db else None
    st = new_status()
    ql.qlinear_bwd_dw(dy_t, xq, sx, dw, db, ws, st)
    assert status_word(st) == 0
    return dw, db, ws


def fwd_magnitude(xq, sx, wq, sw, bias):
    """Summand magnitude of y: |(float)acc * s_x * s_w| + |bias|."""
    acc, _ = oracle.gemm_nt(xq, wq)
    D = np.abs(acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :])
    if bias is not None:
        D = D + np.abs(bias.astype(np.float64))[None, :]
    return D


def layer_inputs(M, K, N, dtype, seed):
    x = workloads.normal((M, K), 1.0, seed)
    x[:, : max(1, K // 100)] *= np.float32(30.0)
    w = workloads.normal((N, K), 0.02, seed + 1)
    b = workloads.normal((N,), 0.01, seed + 2)
    dy = workloads.normal((M, N), 1.0, seed + 3)
    xt = torch.from_numpy(x).to(dtype)
    dyt = torch.from_numpy(dy).to(dtype)
    return xt, w, b, dyt


# ------------------------------------------------------------------ forward
FWD_CASES = [
    # M, K, N, B, in dtype, out dtype
    (32, 256, 128, 256, torch.float32, torch.float32),     # tiny layer
    (300, 384, 272, 128, torch.bfloat16, torch.float32),   # 3x2 tiles, ragged M and N
    (300, 384, 272, 128, torch.bfloat16, torch.bfloat16),
    (129, 1040, 528, 16, torch.float32, torch.bfloat16),   # K tail (1040 = 8*128 + 16)
    (1, 512, 4096, 0, torch.float32, torch.float32),
    (257, 128, 16, 0, torch.bfloat16, torch.float32),      # N = 16, single k-block
]


@pytest.mark.parametrize("M,K,N,B,xt,yt", FWD_CASES)
def test_fwd_parity(M, K, N, B, xt, yt):
    x_t, w, b, _ = layer_inputs(M, K, N, xt, 100 + M + K)
    wq, sw = prep_weight(w, B)
    y, xq, sx = gpu_fwd(dev(x_t), wq, sw, dev(b), B, yt)
    ry, rxq, rsx, rst = oracle.fwd(x_t.float().numpy(), host(wq), host(sw), b, B)
    assert rst == 0
    assert np.array_equal(host(xq), rxq) and np.array_equal(host(sx), rsx)
    D = fwd_magnitude(rxq, rsx, host(wq), host(sw), b)
    assert_close(host(y), ry, D, bf16=(yt == torch.bfloat16), what="y")


@pytest.mark.parametrize("M", [1, 15, 16, 17])
def test_fwd_edge_rows_full_layer(M):
    """Below torch._int_mm's row floor (OneTrainer PR #1681 item 3): M = 1,
    15, 16, 17 on the 5376 -> 7168 layer."""
    d = workloads.rotated_layer(M=M, seed=M, with_dy=False)
    wq, sw = prep_weight(d["w"], 128)
    y, xq, sx = gpu_fwd(dev(d["x_bf16"]), wq, sw, dev(d["bias"]), 128, torch.bfloat16)
    ry, rxq, rsx, _ = oracle.fwd(d["x"], host(wq), host(sw), d["bias"], 128)
    assert np.array_equal(host(xq), rxq) and np.array_equal(host(sx), rsx)
    D = fwd_magnitude(rxq, rsx, host(wq), host(sw), d["bias"])
    assert_close(host(y), ry, D, bf16=True, what="y")


@pytest.mark.parametrize("M,K,N", [(200, 1024, 384),   # CTA-pair tiles
                                   (100, 1024, 384),   # one slab: 64-wide tiles
                                   (1, 5376, 7168),    # up to 4 rows: warp per weight row
                                   (3, 1040, 272), (4, 528, 4096), (16, 528, 4096)])
def test_fwd_int32_accumulator_bit_exact(M, K, N):
    """Unit scales make y the int32 accumulator converted to float: integer
    rows with max |x| = 127 quantize to themselves with s_x = 1."""
    rng = np.random.Generator(np.random.PCG64(7 + M))
    xi = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    xi[:, 0] = 127.0
    wq_np = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    wq = dev(wq_np)
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y, xq, sx = gpu_fwd(dev(xi), wq, sw, None, 0, torch.float32)
    assert np.all(host(sx) == 1.0)
    acc, _ = oracle.gemm_nt(xi.astype(np.int8), wq_np)
    assert np.array_equal(host(y), acc.astype(np.float32))


# ------------------------------------------------------------------ dX
DX_CASES = [
    # M, N (contraction), K (out), B, dy dtype, dx dtype
    (32, 128, 256, 256, torch.float32, torch.float32),     # tiny layer: two-pass rotation
    (32, 128, 256, 256, torch.float32, torch.bfloat16),
    (300, 272, 384, 128, torch.bfloat16, torch.float32),   # fused rotation in the epilogue
    (300, 272, 384, 128, torch.bfloat16, torch.bfloat16),
    (129, 528, 1040, 16, torch.float32, torch.float32),
    (77, 144, 512, 64, torch.float32, torch.float32),
    (33, 400, 272, 0, torch.bfloat16, torch.float32),
]


@pytest.mark.parametrize("M,N,K,B,dyt,dxt", DX_CASES)
def test_bwd_dx_parity(M, N, K, B, dyt, dxt):
    _, w, _, dy_t = layer_inputs(M, K, N, dyt, 200 + M + N)
    wq, sw = prep_weight(w, B)
    dx, ws = gpu_dx(dev(dy_t), wq, sw, B, dxt)
    dy32 = dy_t.float().numpy()
    rdx, rq, rs1, rst = oracle.bwd_dx(dy32, host(wq), host(sw), B)
    assert rst == 0
    # the row-quantized gradient codes and scales in the workspace
    assert np.array_equal(host(ws[: M * N]).view(np.int8).reshape(M, N), rq)
    off = (M * N + 255) // 256 * 256
    assert np.array_equal(host(ws[off: off + 4 * M]).view(np.float32), rs1)
    acc, _ = oracle.gemm_nn(rq, host(wq))
    pre = acc.astype(np.float64) * rs1[:, None]
    D = rotated_magnitude(pre, B) if B else np.abs(pre)
    assert_close(host(dx), rdx, D, bf16=(dxt == torch.bfloat16), what="dX")


@pytest.mark.parametrize("M", [1, 15, 16, 17])
def test_bwd_dx_edge_rows_full_layer(M):
    d = workloads.rotated_layer(M=M, seed=40 + M)
    wq, sw = prep_weight(d["w"], 128)
    dx, _ = gpu_dx(dev(d["dy_bf16"]), wq, sw, 128, torch.bfloat16)
    rdx, rq, rs1, _ = oracle.bwd_dx(d["dy"], host(wq), host(sw), 128)
    acc, _ = oracle.gemm_nn(rq, host(wq))
    D = rotated_magnitude(acc.astype(np.float64) * rs1[:, None], 128)
    assert_close(host(dx), rdx, D, bf16=True, what="dX")


def test_bwd_dx_int32_accumulator_bit_exact():
    rng = np.random.Generator(np.random.PCG64(8))
    M, N, K = 150, 640, 512
    dyi = rng.integers(-127, 128, size=(M, N)).astype(np.float32)
    dyi[:, 1] = -127.0
    wq_np = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    dx, _ = gpu_dx(dev(dyi), dev(wq_np), sw, 0, torch.float32)
    acc, _ = oracle.gemm_nn(dyi.astype(np.int8), wq_np)
    assert np.array_equal(host(dx), acc.astype(np.float32))


# ------------------------------------------------------------------ dW
DW_CASES = [
    # M (contraction), N, K, dy dtype
    (32, 128, 256, torch.float32),      # tiny layer
    (300, 272, 400, torch.bfloat16),    # contraction tail, ragged N and K
    (1, 144, 256, torch.float32),       # contraction of one row
    (15, 256, 512, torch.bfloat16),
    (16, 256, 512, torch.bfloat16),
    (17, 256, 512, torch.bfloat16),
    (1000, 528, 1040, torch.float32),
]


@pytest.mark.parametrize("M,N,K,dyt", DW_CASES)
def test_bwd_dw_parity(M, N, K, dyt):
    x_t, _, _, dy_t = layer_inputs(M, K, N, dyt, 300 + M + N)
    xq_np, sx_np, _ = oracle.quantize_rows(x_t.float().numpy(), B=0)
    dw, db, ws = gpu_dw(dev(dy_t), dev(xq_np), dev(sx_np))
    dy32 = dy_t.float().numpy()
    rdw, rdb, rq, rs2, rst = oracle.bwd_dw(dy32, xq_np, sx_np)
    assert rst == 0
    assert np.array_equal(host(ws[: M * N]).view(np.int8).reshape(M, N), rq)
    acc, _ = oracle.gemm_tn(rq, xq_np)
    assert_close(host(dw), rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")
    assert_close(host(db), rdb, np.abs(dy32.astype(np.float64)).sum(0), what="db")


def test_bwd_dw_int32_accumulator_bit_exact():
    """s_x = 1 and integer dY columns containing 127 make dW the int32
    accumulator of dYq_c^T X_q converted to float."""
    rng = np.random.Generator(np.random.PCG64(9))
    M, N, K = 700, 272, 512
    dyi = rng.integers(-127, 128, size=(M, N)).astype(np.float32)
    dyi[3, :] = 127.0
    xq_np = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    dw, db, _ = gpu_dw(dev(dyi), dev(xq_np), torch.ones(M, device="cuda"))
    acc, _ = oracle.gemm_tn(dyi.astype(np.int8), xq_np)
    assert np.array_equal(host(dw), acc.astype(np.float32))
    assert np.array_equal(host(db), dyi.sum(0).astype(np.float32))


# ------------------------------------------------------------------ combined backward
def gpu_bwd(dy_t, wq, sw, xq, sx, B, dxt):
    M, N = dy_t.shape
    K = wq.shape[1]
    ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, B), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=dxt, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd(dy_t, wq, sw, xq, sx, B, dx, dw, db, ws, st)
    assert status_word(st) == 0
    return dx, dw, db, ws


BWD_CASES = [
    # M, N, K, block, dy dtype, dx dtype
    (32, 128, 256, 256, torch.float32, torch.float32),
    (300, 272, 384, 128, torch.bfloat16, torch.bfloat16),
    (129, 528, 1040, 16, torch.float32, torch.bfloat16),
    (1000, 7168, 256, 0, torch.bfloat16, torch.float32),   # 28 chunks per dY row
    (17, 144, 512, 64, torch.bfloat16, torch.float32),
    (600, 8208, 128, 0, torch.float32, torch.float32),     # > 8192 columns: separate passes
]


@pytest.mark.parametrize("M,N,K,B,dyt,dxt", BWD_CASES)
def test_bwd_combined_matches_oracle_and_separate_calls(M, N, K, B, dyt, dxt):
    x_t, w, _, dy_t = layer_inputs(M, K, N, dyt, 400 + M + N)
    wq, sw = prep_weight(w, B)
    xq_np, sx_np, _ = oracle.quantize_rows(x_t.float().numpy(), B=B)
    xq, sx = dev(xq_np), dev(sx_np)
    dyd = dev(dy_t)
    dx, dw, db, ws = gpu_bwd(dyd, wq, sw, xq, sx, B, dxt)
    # the same results as the two separate calls, bit for bit
    dx1, _ = gpu_dx(dyd, wq, sw, B, dxt)
    dw1, db1, _ = gpu_dw(dyd, xq, sx)
    assert torch.equal(dx, dx1) and torch.equal(dw, dw1) and torch.equal(db, db1)
    dy32 = dy_t.float().numpy()
    rdx, rq, rs1, _ = oracle.bwd_dx(dy32, host(wq), host(sw), B)
    rdw, rdb, rqc, rs2, _ = oracle.bwd_dw(dy32, xq_np, sx_np)
    acc, _ = oracle.gemm_nn(rq, host(wq))
    pre = acc.astype(np.float64) * rs1[:, None]
    assert_close(host(dx), rdx, rotated_magnitude(pre, B) if B else np.abs(pre),
                 bf16=(dxt == torch.bfloat16), what="dX")
    acc, _ = oracle.gemm_tn(rqc, xq_np)
    assert_close(host(dw), rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")
    assert_close(host(db), rdb, np.abs(dy32.astype(np.float64)).sum(0), what="db")


@pytest.mark.parametrize("dyt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
def test_bwd_combined_flags_nonfinite(dyt, bad):
    """One non-finite dY element sets QL_ERR_NONFINITE in the combined
    backward's gradient preparation (NaN through the column sums, +-inf
    through the maxima); the outputs are unspecified."""
    M, N, K, B = 300, 528, 256, 128
    x_t, w, _, dy_t = layer_inputs(M, K, N, dyt, 77)
    wq, sw = prep_weight(w, B)
    xq_np, sx_np, _ = oracle.quantize_rows(x_t.float().numpy(), B=B)
    dy_t = dy_t.clone()
    dy_t[123, 301] = bad
    ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, B), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd(dev(dy_t), wq, sw, dev(xq_np), dev(sx_np), B, dx, dw, db, ws, st)
    assert status_word(st) & (1 << ql.QL_ERR_NONFINITE)


# ------------------------------------------------------------------ full size
def _sample_rows(M, n, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = {0, M - 1, 127, 128} | set(rng.integers(0, M, size=n).tolist())
    return np.array(sorted(r for r in rows if r < M))


@pytest.mark.parametrize("M", [2048, 12000])
def test_full_layer_sampled(M):
    """The 5376 -> 7168 layer at 2048 and 12000 tokens, bf16 X and dY, Hadamard
    block 128, in the launch configuration the benchmark times: all saved
    codes and scales exact; y, dX rows and dW rows sampled against the oracle."""
    d = workloads.rotated_layer(M=M, seed=1)
    B, K, N = 128, d["K"], d["N"]
    wq, sw = prep_weight(d["w"], B)
    wq_np, sw_np = host(wq), host(sw)
    rwq, rsw, _ = oracle.quantize_rows(d["w"], B=B, flags=oracle.REJECT_ZERO_ROWS)
    assert np.array_equal(wq_np, rwq) and np.array_equal(sw_np, rsw)

    bias = dev(d["bias"])
    y, xq, sx = gpu_fwd(dev(d["x_bf16"]), wq, sw, bias, B, torch.bfloat16)
    rxq, rsx, _ = oracle.quantize_rows(d["x"], B=B)
    xq_np, sx_np = host(xq), host(sx)
    assert np.array_equal(xq_np, rxq) and np.array_equal(sx_np, rsx)
    rows = _sample_rows(M, 12, M)
    ry, _, _, _ = oracle.fwd(d["x"][rows], wq_np, sw_np, d["bias"], B)
    D = fwd_magnitude(rxq[rows], rsx[rows], wq_np, sw_np, d["bias"])
    assert_close(host(y)[rows], ry, D, bf16=True, what="y")

    dy_t = dev(d["dy_bf16"])
    dx, ws_dx = gpu_dx(dy_t, wq, sw, B, torch.bfloat16)
    # every row-quantized gradient code and row scale of the input gradient
    rq_all, rs1_all, rst = oracle.bwd_prep_rows(d["dy"], sw_np)
    assert rst == 0
    s1_off = (M * N + 255) // 256 * 256
    assert np.array_equal(host(ws_dx[:M * N]).view(np.int8).reshape(M, N), rq_all)
    assert np.array_equal(host(ws_dx[s1_off: s1_off + 4 * M]).view(np.float32), rs1_all)
    del ws_dx
    rdx, rq, rs1, _ = oracle.bwd_dx(d["dy"][rows], wq_np, sw_np, B)
    acc, _ = oracle.gemm_nn(rq, wq_np)
    assert_close(host(dx)[rows], rdx, rotated_magnitude(acc * rs1[:, None].astype(np.float64), B),
                 bf16=True, what="dX")

    dw, db, ws = gpu_dw(dy_t, xq, sx)
    dx2, dw2, db2, ws2 = gpu_bwd(dy_t, wq, sw, xq, sx, B, torch.bfloat16)
    assert torch.equal(dx2, dx) and torch.equal(dw2, dw) and torch.equal(db2, db)
    # the combined backward's row-quantized codes and scales, all rows
    assert np.array_equal(host(ws2[:M * N]).view(np.int8).reshape(M, N), rq_all)
    assert np.array_equal(host(ws2[s1_off: s1_off + 4 * M]).view(np.float32), rs1_all)
    del ws2, rq_all
    cols = _sample_rows(N, 12, M + 1)
    rdw, rdb, rqc, rs2, _ = oracle.bwd_dw(d["dy"][:, cols], xq_np, sx_np)
    gq = host(ws[: M * N]).view(np.int8).reshape(M, N)
    assert np.array_equal(gq[:, cols], rqc)
    acc, _ = oracle.gemm_tn(rqc, xq_np)
    assert_close(host(dw)[cols], rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")
    assert_close(host(db)[cols], rdb, np.abs(d["dy"][:, cols].astype(np.float64)).sum(0), what="db")


def test_empty_and_degenerate_sizes():
    """M = 0 is a no-op; an empty contraction gives bias / zeros."""
    st = new_status()
    wq = torch.zeros((32, 64), dtype=torch.int8, device="cuda")
    sw = torch.ones(32, device="cuda")
    x0 = torch.zeros((0, 64), device="cuda")
    ql.qlinear_fwd(x0, wq, sw, None, 0, torch.zeros((0, 32), device="cuda"),
                   torch.zeros((0, 64), dtype=torch.int8, device="cuda"),
                   torch.zeros(0, device="cuda"), st)
    # K = 0: y = bias
    x = torch.zeros((5, 0), device="cuda")
    b = torch.arange(32, dtype=torch.float32, device="cuda")
    y = torch.full((5, 32), 7.0, device="cuda")
    ql.qlinear_fwd(x, torch.zeros((32, 0), dtype=torch.int8, device="cuda"), sw, b, 0, y,
                   torch.zeros((5, 0), dtype=torch.int8, device="cuda"),
                   torch.full((5,), 3.0, device="cuda"), st)
    assert torch.equal(y, b.expand(5, 32))
    # M = 0 in the weight gradient: dW = 0, db = 0
    dw = torch.full((32, 64), 5.0, device="cuda")
    db = torch.full((32,), 5.0, device="cuda")
    ws = torch.empty(ql.qlinear_workspace_bytes(0, 32, 64, 0), dtype=torch.uint8, device="cuda")
    ql.qlinear_bwd_dw(torch.zeros((0, 32), device="cuda"),
                      torch.zeros((0, 64), dtype=torch.int8, device="cuda"),
                      torch.zeros(0, device="cuda"), dw, db, ws, st)
    assert not dw.any() and not db.any()
    assert status_word(st) == 0
