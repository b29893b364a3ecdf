"""GPU parity of the forward's bf16 route (OneTrainer PR #1681, third commit
note: rotate the activations, do not quantize them, multiply on bf16 tensor
cores) against the oracle, through the C ABI.  The rotated bf16 activations
are compared bit for bit; y within the bound of float32 accumulation (1e-3
of the summand magnitude, plus half a bf16 ulp for bf16 outputs).  The
full-size case also reproduces the page's comparison of the two routes
against the dequantized weight."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import assert_close, dev, host, new_status, status_word

pytestmark = pytest.mark.gpu


def _codes_bf16(q_np):
    wq = dev(q_np)
    out = torch.empty(wq.shape, dtype=torch.bfloat16, device="cuda")
    ql.qlinear_codes_bf16(wq, out)
    return out


def _route(x_t, wb, sw, bias, B, yt):
    M, K = x_t.shape
    N = wb.shape[0]
    nbytes = ql.qlinear_fwd_bf16_workspace_bytes(M, K, x_t.dtype, B)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda") if nbytes else None
    y = torch.empty((M, N), dtype=yt, device="cuda")
    st = new_status()
    ql.qlinear_fwd_bf16(x_t, wb, sw, bias, B, y, ws, st)
    assert status_word(st) == 0
    return y, ws


CASES = [
    # M, K, N, B, x dtype, y dtype
    (1, 256, 128, 0, torch.float32, torch.float32),
    (17, 5376, 272, 128, torch.bfloat16, torch.bfloat16),
    (300, 1040, 528, 16, torch.float32, torch.bfloat16),   # K tail: 1040 = 16 * 65
    (129, 384, 256, 128, torch.bfloat16, torch.float32),
    (257, 512, 16, 0, torch.bfloat16, torch.float32),      # bf16 x, no rotation: no workspace
    (600, 2048, 1000 // 16 * 16, 256, torch.float32, torch.float32),
]


@pytest.mark.parametrize("M,K,N,B,xt,yt", CASES)
def test_bf16_route_matches_oracle(M, K, N, B, xt, yt):
    x = workloads.normal((M, K), 1.0, M + K)
    x[:, : max(1, K // 100)] *= np.float32(30.0)
    x_t = torch.from_numpy(x).to(xt)
    x32 = x_t.float().numpy()
    w = workloads.normal((N, K), 0.02, N + 1)
    b = workloads.normal((N,), 0.01, N + 2)
    q, s, _ = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
    wb = _codes_bf16(q)
    assert np.array_equal(host(wb), q.astype(np.float32))
    y, ws = _route(dev(x_t), wb, dev(s), dev(b), B, yt)
    ry, rxr, st = oracle.fwd_bf16(x32, q, s, b, B)
    assert st == 0
    if ws is not None:
        xr = ws[: 2 * M * K].view(torch.bfloat16).view(M, K)
        assert np.array_equal(host(xr), rxr)
    D = (np.abs(rxr.astype(np.float64)) @ np.abs(q.astype(np.float64)).T) * s[None, :] + np.abs(b)
    assert_close(host(y), ry, D, bf16=(yt == torch.bfloat16), what="y (bf16 route)")


def test_bf16_route_empty_contraction_gives_bias():
    x = torch.zeros((5, 0), dtype=torch.bfloat16, device="cuda")
    wb = torch.zeros((32, 0), dtype=torch.bfloat16, device="cuda")
    b = torch.arange(32, dtype=torch.float32, device="cuda")
    y = torch.full((5, 32), 7.0, device="cuda")
    st = new_status()
    ql.qlinear_fwd_bf16(x, wb, torch.ones(32, device="cuda"), b, 0, y, None, st)
    assert status_word(st) == 0 and torch.equal(y, b.expand(5, 32))


@pytest.mark.slow
def test_routes_against_the_dequantized_weight():
    """The 5376 -> 7168 layer at 2048 tokens, block 128: both forward routes
    against Y* = x W_hat^T + b in float64, W_hat the dequantized weight in the
    original basis.  The bf16 route skips the activation quantization, so it
    must be the more accurate one (the page measures 3.61e-3 against
    9.43e-3 on its own data); its sampled rows also match the oracle."""
    d = workloads.rotated_layer(M=2048, seed=1)
    B, N = 128, d["N"]
    q, s, _ = oracle.quantize_rows(d["w"], B=B, flags=oracle.REJECT_ZERO_ROWS)
    wq, sw, bias = dev(q), dev(s), dev(d["bias"])
    x_t = dev(d["x_bf16"])
    M, K = x_t.shape
    y8 = torch.empty((M, N), device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    st = new_status()
    ql.qlinear_fwd(x_t, wq, sw, bias, B, y8, xq, sx, st)
    assert status_word(st) == 0
    yb, _ = _route(x_t, _codes_bf16(q), sw, bias, B, torch.float32)
    rows = np.array(sorted(set(np.random.Generator(np.random.PCG64(7)).integers(0, M, 48).tolist())))
    w_hat, _ = oracle.dequantize(q, s, B)
    ystar = d["x"][rows].astype(np.float64) @ w_hat.astype(np.float64).T + d["bias"]
    ri = torch.from_numpy(rows).cuda()
    e8 = np.linalg.norm(host(y8[ri]) - ystar) / np.linalg.norm(ystar)
    eb = np.linalg.norm(host(yb[ri]) - ystar) / np.linalg.norm(ystar)
    print(f"relative error vs dequantized weight: int8 route {e8:.3e}, bf16 route {eb:.3e}")
    assert eb < e8
    ry, rxr, _ = oracle.fwd_bf16(d["x"][rows], q, s, d["bias"], B)
    D = (np.abs(rxr.astype(np.float64)) @ np.abs(q.astype(np.float64)).T) * s[None, :] + np.abs(d["bias"])
    assert_close(host(yb[ri]), ry, D, what="y (bf16 route, 2048 tokens)")
