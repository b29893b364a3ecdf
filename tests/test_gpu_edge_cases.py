"""The method's edge cases through the kernels that the full-size layer calls
take, against the oracle, through the C ABI: all-zero rows (with and without
QL_REJECT_ZERO_ROWS), all-zero gradient columns, a zero saved-input scale, a
single NaN, +inf or -inf, finite values whose float32 partial sums overflow,
and rows built so that t * (127 / amax) lands exactly on k + 1/2 for many k
(round-to-nearest-even ties, decided on the GPU through the float adder).

Shapes are those of the 5376-wide layer at several hundred tokens, where the
activation quantizer runs its persistent bf16 block-128 path, the row
quantization of a wide fp32 or bf16 matrix its staged path, and the combined
backward its streamed gradient preparation.  Codes, scales and the status
word are compared bit for bit; where a non-finite value makes a row or column
unspecified, every other row or column is still compared."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import assert_close, dev, host, new_status, status_word

pytestmark = pytest.mark.gpu

NONFINITE = 1 << ql.QL_ERR_NONFINITE
ZERO_ROW = 1 << ql.QL_ERR_ZERO_ROW


def _a256(n: int) -> int:
    return (n + 255) // 256 * 256


# ------------------------------------------------------------------ tie rows
def _bf16_head(v: np.float32) -> np.float32:
    """v truncated to its top 8 significant bits (a bf16 value)."""
    return np.array([v], np.float32).view(np.uint32).__and__(np.uint32(0xFFFF0000)).view(np.float32)[0]


def _split3(S: np.float32):
    """S = a + b + c exactly with a, b, c bf16 values, or None."""
    a = _bf16_head(S)
    r = np.float32(S - a)
    b = _bf16_head(r)
    c = np.float32(r - b)
    if _bf16_head(c) != c or np.float32(np.float32(a + b) + c) != S:
        return None
    return a, b, c


def _tie_sums(c: np.float32, inv: np.float32):
    """For each k in 0..126 that has one: three bf16 values whose exact float32
    sum S has fl32(fl32(S * c) * inv) == k + 1/2.  (Not every k has such an S:
    consecutive float32 S can step fl32(S * c) by more than one ulp.)"""
    table = {}
    for k in range(127):
        v = np.float32(k + 0.5)
        S0 = np.float32(float(v) / float(inv) / float(c))
        for n in range(256):
            hit = None
            for sg in (1, -1):
                S = np.float32(S0 + sg * n * np.spacing(S0))
                if np.float32(np.float32(S * c) * inv) == v:
                    hit = _split3(S)
                    if hit is not None:
                        break
            if hit is not None:
                table[k] = hit
                break
    return table


def tie_rows(rows: int, cols: int, B: int, seed: int) -> np.ndarray:
    """Rows whose values after the block-Hadamard of width B (none for B = 0)
    make t * (127 / amax) land exactly on k + 1/2 for many elements (ties).

    B = 0: values k + 1/2 and one 127 per row, so 127 / amax = 1.  B > 0: one
    block per row holds the single value 1000 (bf16-exact), whose rotation
    sets amax = fl32(1000 * c) with c = fl32(1/sqrt(B)), hence inv =
    fl32(127 / amax); each other block holds x[0] + x[1] + x[2] = S (three
    bf16 values, so the butterflies' sums are exact) with fl32(fl32(S * c) *
    inv) = k + 1/2, which every output j of the block with j % 4 == 0 then
    reaches; the block's other outputs are smaller and not ties."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = np.zeros((rows, cols), np.float32)
    if B == 0:
        k = rng.integers(0, 127, size=(rows, cols)).astype(np.float32)
        sign = np.where(rng.integers(0, 2, size=(rows, cols)) == 1, -1.0, 1.0).astype(np.float32)
        x[:] = sign * (k + np.float32(0.5))
        x[np.arange(rows), rng.integers(0, cols, size=rows)] = 127.0
        return x
    c = np.float32(oracle.hadamard_scale(B))
    top_value = np.float32(1000.0)
    inv = np.float32(np.float32(127.0) / np.float32(top_value * c))
    table = _tie_sums(c, inv)
    ks = np.array(sorted(table))
    assert (ks % 2 == 0).sum() >= 20 and (ks % 2 == 1).sum() >= 20
    nblk = cols // B
    for r in range(rows):
        top = int(rng.integers(0, nblk))
        pick = rng.integers(0, len(ks), size=nblk)
        flip = rng.integers(0, 2, size=nblk)
        for b in range(nblk):
            if b == top:
                x[r, b * B] = top_value
            else:
                sg = np.float32(-1.0 if flip[b] else 1.0)
                x[r, b * B: b * B + 3] = [sg * v for v in table[int(ks[pick[b]])]]
    return x


def _count_ties(x32: np.ndarray, B: int) -> int:
    """How many rotated values of x sit exactly on k + 1/2 (the test's own
    check that the construction produced ties)."""
    t = oracle.hadamard_rows(x32, B)[0] if B else x32
    amax = np.abs(t).max(axis=1, keepdims=True)
    v = (t * (np.float32(127.0) / amax).astype(np.float32)).astype(np.float32)
    return int((np.abs(v - np.floor(v)) == 0.5).sum())


# ------------------------------------------------------------------ quantizer
def _quant(x_t, B, flags=0):
    rows, cols = x_t.shape
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_quantize_rows(x_t, q, s, st, hadamard_block=B, flags=flags)
    return host(q), host(s), status_word(st)


# rows, cols, block, dtype: the persistent bf16 block-128 path (the forward's
# input at >= 4 rows per SM), its block-0 form, and the staged row paths
QUANT_PATHS = [
    (640, 5376, 128, torch.bfloat16),
    (700, 4096, 0, torch.bfloat16),
    (400, 5376, 128, torch.bfloat16),
    (400, 2320, 16, torch.float32),
]


@pytest.mark.parametrize("rows,cols,B,dtype", QUANT_PATHS)
def test_quantizer_exact_ties(rows, cols, B, dtype):
    if B == 16:  # fl32(1/4) is exact: the rows' block sums give the targets directly
        x = np.zeros((rows, cols), np.float32)
        base = tie_rows(rows, cols // 16, 0, rows + cols)
        x[:, ::16] = base * np.float32(4.0)
    else:
        x = tie_rows(rows, cols, B, rows + cols)
    xt = torch.from_numpy(x).to(dtype)
    x32 = xt.float().numpy()
    assert np.array_equal(x32, x)  # every value is exact in the input dtype
    assert _count_ties(x32, B) >= rows * cols // 8
    q, s, st = _quant(dev(xt), B)
    rq, rs, rst = oracle.quantize_rows(x32, B=B)
    assert st == rst == 0
    assert np.array_equal(s, rs)
    assert np.array_equal(q, rq)


@pytest.mark.parametrize("rows,cols,B,dtype", QUANT_PATHS)
def test_quantizer_zero_rows(rows, cols, B, dtype):
    x = workloads.normal((rows, cols), 1.0, rows + 3 * cols)
    zero = [0, 5, rows // 2, rows - 1]
    x[zero] = 0.0
    xt = torch.from_numpy(x).to(dtype)
    x32 = xt.float().numpy()
    for flags in (0, ql.QL_REJECT_ZERO_ROWS):
        q, s, st = _quant(dev(xt), B, flags)
        rq, rs, rst = oracle.quantize_rows(x32, B=B, flags=flags)
        assert st == rst == (ZERO_ROW if flags else 0)
        assert np.array_equal(s, rs) and np.array_equal(q, rq)
        assert not s[zero].any() and not q[zero].any()


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("rows,cols,B,dtype", QUANT_PATHS)
def test_quantizer_single_nonfinite(rows, cols, B, dtype, bad):
    x = workloads.normal((rows, cols), 1.0, rows + 5 * cols)
    r0, c0 = rows // 3, cols - 37
    x[r0, c0] = bad
    xt = torch.from_numpy(x).to(dtype)
    x32 = xt.float().numpy()
    q, s, st = _quant(dev(xt), B)
    rq, rs, rst = oracle.quantize_rows(x32, B=B)
    assert rst == NONFINITE and st == rst
    keep = np.arange(rows) != r0  # the bad row's codes and scale are unspecified
    assert np.array_equal(s[keep], rs[keep]) and np.array_equal(q[keep], rq[keep])


# ------------------------------------------------------------------ backward
M_BWD, N_BWD, K_BWD = 640, 5376, 256


def _ws_offsets(M, N, K, B):
    """Where the backward calls leave their int8 gradient copies and scales
    in the workspace: the row-quantized (or, for the weight-gradient call
    alone, column-quantized) codes first, then s' [M], the column maxima [N],
    s'' [N]; qlinear_bwd puts the column-quantized codes after the common
    layout, whose size qlinear_workspace_bytes reports."""
    s1 = _a256(M * N)
    s2 = s1 + _a256(4 * M) + _a256(4 * N)
    return {"codes": 0, "s1": s1, "s2": s2, "codes_c": ql.qlinear_workspace_bytes(M, N, K, B)}


def _ws_codes(ws, off, M, N):
    return host(ws[off: off + M * N]).view(np.int8).reshape(M, N)


def _ws_f32(ws, off, n):
    return host(ws[off: off + 4 * n]).view(np.float32)


def bwd_tie_inputs(seed):
    """dY with exact ties in both quantizations of the backward: s_w = 0.5,
    so the row maxima of |dY * s_w| are 63.5 (column 0 holds +-127) and
    127 / 63.5 = 2 makes (dY * 0.5) * 2 = dY; s_x = 1 (and 0 on two rows), so
    the column maxima of |dY * s_x| are 127 (row 0 holds 127) and the codes
    are rne(dY).  dY is +-(k + 1/2) elsewhere, all exact in bf16; one dY row
    and one dY column are all zero."""
    M, N, K = M_BWD, N_BWD, K_BWD
    rng = np.random.Generator(np.random.PCG64(seed))
    dy = tie_rows(M, N, 0, seed)
    dy[:, 0] = np.where(rng.integers(0, 2, size=M) == 1, -127.0, 127.0)
    dy[0, :] = 127.0
    dy[11, :] = 0.0            # a zero gradient row: s' = 0, zero codes
    dy[:, 17] = 0.0            # a zero gradient column: s'' = 0, zero codes
    sw = np.full(N, 0.5, np.float32)
    sx = np.ones(M, np.float32)
    sx[[7, 300]] = 0.0         # zero rows of the saved input
    wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    xq[[7, 300]] = 0
    return dy, sw, sx, wq, xq


def _run_bwd(dy_t, sw, sx, wq, xq, B=0):
    M, N = dy_t.shape
    K = wq.shape[1]
    ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, B), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd(dev(dy_t), dev(wq), dev(sw), dev(xq), dev(sx), B, dx, dw, db, ws, st)
    return ws, dx, dw, db, status_word(st)


@pytest.mark.parametrize("dyt", [torch.bfloat16, torch.float32])
def test_bwd_combined_ties_and_zero_rows_columns(dyt):
    dy, sw, sx, wq, xq = bwd_tie_inputs(21)
    M, N, K = dy.shape + (wq.shape[1],)
    dy_t = torch.from_numpy(dy).to(dyt)
    assert np.array_equal(dy_t.float().numpy(), dy)
    ws, dx, dw, db, st = _run_bwd(dy_t, sw, sx, wq, xq)
    rdx, rq, rs1, rst1 = oracle.bwd_dx(dy, wq, sw)
    rdw, rdb, rqc, rs2, rst2 = oracle.bwd_dw(dy, xq, sx)
    assert st == (rst1 | rst2) == 0
    off = _ws_offsets(M, N, K, 0)
    assert np.array_equal(_ws_f32(ws, off["s1"], M), rs1) and rs1[11] == 0
    assert np.array_equal(_ws_codes(ws, off["codes"], M, N), rq)
    assert np.array_equal(_ws_f32(ws, off["s2"], N), rs2) and rs2[17] == 0
    assert np.array_equal(_ws_codes(ws, off["codes_c"], M, N), rqc)
    # every partial sum of the k + 1/2 values is exact, so db is too
    assert np.array_equal(host(db), rdb)
    assert not host(dw)[17].any() and not host(dx)[11].any()
    acc, _ = oracle.gemm_nn(rq, wq)
    assert_close(host(dx), rdx, np.abs(acc.astype(np.float64) * rs1[:, None]), what="dX")
    acc, _ = oracle.gemm_tn(rqc, xq)
    assert_close(host(dw), rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")


def test_bwd_separate_calls_ties_and_zero_rows_columns():
    """The same inputs through qlinear_bwd_dx (row quantization of dY * s_w
    by the staged row kernel) and qlinear_bwd_dw (column statistics and
    column codes alone)."""
    dy, sw, sx, wq, xq = bwd_tie_inputs(22)
    M, N, K = dy.shape + (wq.shape[1],)
    dy_d = dev(torch.from_numpy(dy).to(torch.bfloat16))
    off = _ws_offsets(M, N, K, 0)
    ws = torch.empty(ql.qlinear_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device="cuda")
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dx(dy_d, dev(wq), dev(sw), 0, dx, ws, st)
    rdx, rq, rs1, rst = oracle.bwd_dx(dy, wq, sw)
    assert status_word(st) == rst == 0
    assert np.array_equal(_ws_f32(ws, off["s1"], M), rs1)
    assert np.array_equal(_ws_codes(ws, off["codes"], M, N), rq)
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    db = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dw(dy_d, dev(xq), dev(sx), dw, db, ws, st)
    rdw, rdb, rqc, rs2, rst = oracle.bwd_dw(dy, xq, sx)
    assert status_word(st) == rst == 0
    assert np.array_equal(_ws_f32(ws, off["s2"], N), rs2)
    assert np.array_equal(_ws_codes(ws, off["codes"], M, N), rqc)
    assert np.array_equal(host(db), rdb)
    acc, _ = oracle.gemm_tn(rqc, xq)
    assert_close(host(dw), rdw, np.abs(acc.astype(np.float64) * rs2[:, None]), what="dW")


BAD_SPOTS = [
    # (row, column): an ordinary element, and one in a row whose s_x is 0,
    # where dY * s_x is NaN for an infinite dY
    (123, 301),
    (7, 50),
]


@pytest.mark.parametrize("spot", BAD_SPOTS)
@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
def test_bwd_nonfinite_status_matches_oracle(bad, spot):
    """Combined backward and the weight-gradient call alone: the status word
    equals the oracle's (QL_ERR_NONFINITE exactly when a product dY * s_x or
    dY * s_w is not finite); the codes and scales of every row and column
    that does not hold the bad value are still exact."""
    dy, sw, sx, wq, xq = bwd_tie_inputs(23)
    M, N, K = dy.shape + (wq.shape[1],)
    r0, c0 = spot
    dy[r0, c0] = bad
    dy_t = torch.from_numpy(dy)
    ws, _, _, _, st = _run_bwd(dy_t, sw, sx, wq, xq)
    _, rq, rs1, rst1 = oracle.bwd_dx(dy, wq, sw)
    _, _, rqc, rs2, rst2 = oracle.bwd_dw(dy, xq, sx)
    assert rst2 == NONFINITE and st == (rst1 | rst2)
    off = _ws_offsets(M, N, K, 0)
    rows = np.arange(M) != r0
    cols = np.arange(N) != c0
    assert np.array_equal(_ws_f32(ws, off["s1"], M)[rows], rs1[rows])
    assert np.array_equal(_ws_codes(ws, off["codes"], M, N)[rows], rq[rows])
    assert np.array_equal(_ws_f32(ws, off["s2"], N)[cols], rs2[cols])
    assert np.array_equal(_ws_codes(ws, off["codes_c"], M, N)[:, cols], rqc[:, cols])
    # the weight-gradient call alone flags the same condition
    ws1 = torch.empty(ql.qlinear_workspace_bytes(M, N, K, 0), dtype=torch.uint8, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    st1 = new_status()
    ql.qlinear_bwd_dw(dev(dy_t), dev(xq), dev(sx), dw, None, ws1, st1)
    assert status_word(st1) == rst2
    assert np.array_equal(_ws_f32(ws1, off["s2"], N)[cols], rs2[cols])


def test_bwd_finite_overflowing_partial_sums_are_not_flagged():
    """Finite dY whose float32 column partial sums overflow (two values of
    3e38 in one column) is not a non-finite input: no product dY * s_x or
    dY * s_w leaves the float range, so neither the oracle nor the kernels
    set QL_ERR_NONFINITE; the column's bias gradient is then outside the
    float range and unspecified."""
    dy, sw, sx, wq, xq = bwd_tie_inputs(24)
    M, N, K = dy.shape + (wq.shape[1],)
    dy[[1, 2, 3], 40] = np.float32(3e38)
    ws, _, _, _, st = _run_bwd(torch.from_numpy(dy), sw, sx, wq, xq)
    _, rq, rs1, rst1 = oracle.bwd_dx(dy, wq, sw)
    _, _, rqc, rs2, rst2 = oracle.bwd_dw(dy, xq, sx)
    assert st == (rst1 | rst2) == 0
    off = _ws_offsets(M, N, K, 0)
    assert np.array_equal(_ws_f32(ws, off["s2"], N), rs2)
    assert np.array_equal(_ws_codes(ws, off["codes_c"], M, N), rqc)
    assert np.array_equal(_ws_f32(ws, off["s1"], M), rs1)
    assert np.array_equal(_ws_codes(ws, off["codes"], M, N), rq)
