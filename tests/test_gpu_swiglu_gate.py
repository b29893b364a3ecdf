"""GPU parity of the SwiGLU gate kernels against the oracle, through the C
ABI, on shapes that span several 3584-column pieces with a ragged last one:
the fused gate + quantization of the second projection's input (codes,
scales and status bit for bit), the gate's backward (bit for bit, float32
and bf16 outputs), special values (a = +-0, +-100, beyond the float32 range
of e^-a, NaN and infinities), zero rows, and the forward from the quantized
input against the whole forward."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, host, new_status, status_word

pytestmark = pytest.mark.gpu


def _ab(M, F, seed, dtype):
    d = workloads.swiglu_gate_inputs(T=M, d_ff=F, seed=seed)
    ab = d["ab"].copy()
    ab[0, :6] = np.float32([0.0, -0.0, 100.0, -100.0, -120.0, 95.0])
    t = torch.from_numpy(ab).to(dtype)
    return t, t.float().numpy(), d


def _gate(ab_t, pitch_pad=0):
    M, F2 = ab_t.shape
    F = F2 // 2
    if pitch_pad:
        big = torch.zeros((M, F2 + pitch_pad), dtype=ab_t.dtype)
        big[:, :F2] = ab_t
        src = dev(big)[:, :F2]
    else:
        src = dev(ab_t)
    hq = torch.empty((M, F), dtype=torch.int8, device="cuda")
    sh = torch.empty(M, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_swiglu_quantize(src, hq, sh, st)
    return host(hq), host(sh), status_word(st)


SHAPES = [
    # M, F (pieces of 3584 columns): one ragged piece, two with a ragged
    # second, three whose last holds 16 columns, the MLP's d_ff (four full
    # pieces), the smallest and largest F
    (37, 144), (300, 2064), (129, 6160), (50, 7184), (64, 14336), (3, 16), (1, 16384),
]


@pytest.mark.parametrize("M,F", SHAPES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gate_quantize_bit_exact(M, F, dtype):
    ab_t, ab32, _ = _ab(M, F, M + F, dtype)
    q, s, st = _gate(ab_t)
    rq, rs, rst = oracle.swiglu_quantize(ab32)
    assert st == rst == 0
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


def test_gate_quantize_strided_input_and_zero_rows():
    M, F = 200, 2064
    ab_t, ab32, _ = _ab(M, F, 5, torch.bfloat16)
    ab_t[7, :F] = 0.0       # a = 0: h = 0
    ab_t[9, F:] = 0.0       # b = 0: h = 0
    ab32 = ab_t.float().numpy()
    q, s, st = _gate(ab_t, pitch_pad=32)
    rq, rs, rst = oracle.swiglu_quantize(ab32)
    assert st == rst == 0 and s[7] == 0 and s[9] == 0 and not q[[7, 9]].any()
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("where", ["a", "b"])
def test_gate_quantize_nonfinite(bad, where):
    M, F = 160, 6160
    ab_t, _, _ = _ab(M, F, 6, torch.float32)
    r0 = 77
    ab_t[r0, (0 if where == "a" else F) + 1234] = bad
    ab32 = ab_t.numpy()
    q, s, st = _gate(ab_t)
    rq, rs, rst = oracle.swiglu_quantize(ab32)
    # silu(+inf) * b = inf * b and silu(-inf) = -0: the row may or may not be
    # non-finite; the status must be the oracle's either way
    assert st == rst
    keep = np.arange(M) != r0
    assert np.array_equal(s[keep], rs[keep]) and np.array_equal(q[keep], rq[keep])
    if rst == 0:
        assert np.array_equal(s, rs) and np.array_equal(q, rq)


@pytest.mark.parametrize("M,F", [(37, 144), (300, 2064), (64, 14336)])
@pytest.mark.parametrize("abt,dht,dabt", [
    (torch.bfloat16, torch.bfloat16, torch.bfloat16),
    (torch.bfloat16, torch.float32, torch.float32),
    (torch.float32, torch.bfloat16, torch.bfloat16),
])
def test_gate_bwd_bit_exact(M, F, abt, dht, dabt):
    ab_t, ab32, d = _ab(M, F, 2 * M + F, abt)
    dh_t = torch.from_numpy(d["dh"]).to(dht)
    dab = torch.empty((M, 2 * F), dtype=dabt, device="cuda")
    ql.qlinear_swiglu_bwd(dev(ab_t), dev(dh_t), dab)
    ref = torch.from_numpy(oracle.swiglu_bwd(ab32, dh_t.float().numpy())).to(dabt)
    assert torch.equal(dab.cpu(), ref)


def test_fwd_quantized_equals_the_forward():
    """Given the codes and scales the forward's own quantization writes, the
    forward from codes gives the forward's output bit for bit."""
    M, K, N = 300, 1040, 528
    x = torch.from_numpy(workloads.normal((M, K), 1.0, 8)).to(torch.bfloat16)
    w = workloads.normal((N, K), 0.02, 9)
    b = dev(workloads.normal((N,), 0.01, 10))
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_quantize_rows(dev(w), wq, sw, st, flags=ql.QL_REJECT_ZERO_ROWS)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    ql.qlinear_fwd(dev(x), wq, sw, b, 0, y, xq, sx, st)
    y2 = torch.empty_like(y)
    ql.qlinear_fwd_quantized(xq, sx, wq, sw, b, y2, st)
    assert status_word(st) == 0
    assert torch.equal(y, y2)
    ry, rst = oracle.fwd_quantized(host(xq), host(sx), host(wq), host(sw), host(b))
    assert rst == 0
    assert np.abs(host(y2) - ry).max() <= 2.0 ** -8 * np.abs(ry).max()


def test_gate_validation():
    ab = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")   # F = 24: not a multiple of 16
    hq = torch.zeros((4, 32), dtype=torch.int8, device="cuda")
    sh = torch.zeros(4, device="cuda")
    st = new_status()
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_swiglu_quantize(ab, hq, sh, st)
    assert e.value.code == ql.QL_ERR_SHAPE
    ab = torch.zeros((2, 2 * 16400), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_swiglu_quantize(ab, torch.zeros((2, 16400), dtype=torch.int8, device="cuda"),
                                   sh, st)
    assert e.value.code == ql.QL_ERR_UNSUPPORTED
    assert status_word(st) == 0

