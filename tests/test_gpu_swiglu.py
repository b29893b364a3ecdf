"""GPU parity of the SwiGLU MLP at full size: 8192 tokens, d_model 4096,
d_ff 14336, bf16 activations and gradients, no rotation.

w1 and w3 act on the same input, so they are stacked into one [2*d_ff,
d_model] weight and X is quantized once for both; with per-row weight
scales the stacked call gives exactly the two separate calls' outputs
(checked below).  The gate h = silu(a) * b runs fused with the second
projection's input quantization (qlinear_swiglu_quantize: h codes and
scales bit for bit against the oracle at full size), the second projection
takes those codes (qlinear_fwd_quantized), and the gate's backward
(qlinear_swiglu_bwd: bit for bit) gives the stacked projection's output
gradient.  Each call is checked against the oracle on seeded inputs: saved
codes and scales in full and bit for bit, float outputs on sampled rows (and
sampled weight-gradient rows) within the 1e-3 relative bound plus half a
bf16 ulp."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import assert_close, dev, host, new_status, status_word

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

T, D, F = 8192, 4096, 14336


def _rows(n_total, n, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.array(sorted({0, n_total - 1, 127, 128} | set(rng.integers(0, n_total, n).tolist())))


@pytest.fixture(scope="module")
def mlp():
    return workloads.swiglu_mlp(T=T, d_model=D, d_ff=F, seed=0)


@pytest.fixture(scope="module")
def gate():
    return workloads.swiglu_gate_inputs(T=T, d_ff=F, seed=0)


def _prep(w):
    """Weight codes and scales from the oracle (inputs of the GPU calls)."""
    q, s, st = oracle.quantize_rows(w, flags=oracle.REJECT_ZERO_ROWS)
    assert st == 0
    return q, s


def _fwd(x_t, wq, sw):
    M, K = x_t.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_fwd(x_t, wq, sw, None, 0, y, xq, sx, st)
    assert status_word(st) == 0
    return y, xq, sx


def _bwd(dy_t, wq, sw, xq, sx):
    M, N = dy_t.shape
    K = wq.shape[1]
    ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd(dy_t, wq, sw, xq, sx, 0, dx, dw, db, ws, st)
    assert status_word(st) == 0
    return dx, dw, db


def _check_fwd(x32, y, xq, sx, wq_np, sw_np, seed):
    rxq, rsx, _ = oracle.quantize_rows(x32)
    assert np.array_equal(host(xq), rxq) and np.array_equal(host(sx), rsx)
    rows = _rows(x32.shape[0], 10, seed)
    ry, _, _, _ = oracle.fwd(x32[rows], wq_np, sw_np, None, 0)
    acc, _ = oracle.gemm_nt(rxq[rows], wq_np)
    Dm = np.abs(acc.astype(np.float64) * rsx[rows, None].astype(np.float64) * sw_np[None, :])
    assert_close(host(y[torch.from_numpy(rows).cuda()]), ry, Dm, bf16=True, what="y")
    return rxq, rsx


def _check_bwd(dy32, dx, dw, db, wq_np, sw_np, xq_np, sx_np, seed):
    rows = _rows(dy32.shape[0], 10, seed)
    rdx, rq, rs1, _ = oracle.bwd_dx(dy32[rows], wq_np, sw_np, 0)
    acc, _ = oracle.gemm_nn(rq, wq_np)
    assert_close(host(dx[torch.from_numpy(rows).cuda()]), rdx,
                 np.abs(acc.astype(np.float64) * rs1[:, None]), bf16=True, what="dX")
    cols = _rows(dy32.shape[1], 10, seed + 1)
    rdw, rdb, rqc, rs2, _ = oracle.bwd_dw(np.ascontiguousarray(dy32[:, cols]), xq_np, sx_np)
    acc, _ = oracle.gemm_tn(rqc, xq_np)
    ci = torch.from_numpy(cols).cuda()
    assert_close(host(dw[ci]), rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")
    assert_close(host(db[ci]), rdb, np.abs(dy32[:, cols].astype(np.float64)).sum(0), what="db")


def test_stacked_w13_forward_and_backward(mlp, gate):
    w13 = np.concatenate([mlp["w1"], mlp["w3"]], axis=0)
    wq_np, sw_np = _prep(w13)
    wq, sw = dev(wq_np), dev(sw_np)
    x_t = dev(mlp["x_bf16"])
    y13, xq, sx = _fwd(x_t, wq, sw)
    xq_np, sx_np = _check_fwd(mlp["x"], y13, xq, sx, wq_np, sw_np, 1)
    # the stacked call equals separate w1 and w3 calls, bit for bit
    y1, xq1, sx1 = _fwd(x_t, wq[:F], sw[:F])
    y3, _, _ = _fwd(x_t, wq[F:], sw[F:])
    assert torch.equal(y1, y13[:, :F]) and torch.equal(y3, y13[:, F:])
    assert torch.equal(xq1, xq) and torch.equal(sx1, sx)
    del y13, y1, y3
    # the output gradient [da | db] from the gate's backward (bit for bit
    # against the oracle, then the stacked projection's backward on it)
    dab = torch.empty((T, 2 * F), dtype=torch.bfloat16, device="cuda")
    ql.qlinear_swiglu_bwd(dev(gate["ab_bf16"]), dev(gate["dh_bf16"]), dab)
    rdab = oracle.swiglu_bwd(gate["ab"], gate["dh"])
    rdab_bf = torch.from_numpy(rdab).to(torch.bfloat16)
    assert torch.equal(dab.cpu(), rdab_bf)
    dy13 = rdab_bf.float().numpy()
    del rdab, rdab_bf
    dx, dw, db = _bwd(dab, wq, sw, xq, sx)
    _check_bwd(dy13, dx, dw, db, wq_np, sw_np, xq_np, sx_np, 2)


def test_gate_and_w2_forward_and_backward(mlp, gate):
    wq_np, sw_np = _prep(mlp["w2"])
    wq, sw = dev(wq_np), dev(sw_np)
    hq = torch.empty((T, F), dtype=torch.int8, device="cuda")
    sh = torch.empty(T, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_swiglu_quantize(dev(gate["ab_bf16"]), hq, sh, st)
    assert status_word(st) == 0
    rhq, rsh, rst = oracle.swiglu_quantize(gate["ab"])
    assert rst == 0
    hq_np, sh_np = host(hq), host(sh)
    assert np.array_equal(sh_np, rsh) and np.array_equal(hq_np, rhq)
    y = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    st = new_status()
    ql.qlinear_fwd_quantized(hq, sh, wq, sw, None, y, st)
    assert status_word(st) == 0
    rows = _rows(T, 10, 3)
    ry, _ = oracle.fwd_quantized(rhq[rows], rsh[rows], wq_np, sw_np)
    acc, _ = oracle.gemm_nt(rhq[rows], wq_np)
    Dm = np.abs(acc.astype(np.float64) * rsh[rows, None].astype(np.float64) * sw_np[None, :])
    assert_close(host(y[torch.from_numpy(rows).cuda()]), ry, Dm, bf16=True, what="y")
    del y
    dx, dw, db = _bwd(dev(mlp["dy_bf16"]), wq, sw, hq, sh)
    _check_bwd(mlp["dy"], dx, dw, db, wq_np, sw_np, hq_np, sh_np, 4)
