"""GPU parity of the row kernels against the oracle, through the C ABI:
per-row quantization (optionally scaled per column and rotated) and the
standalone block-Hadamard.  Codes and scales must be bit-exact; the float32
rotation uses the oracle's butterfly order, so it is bit-exact too."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, host, new_status, status_word

pytestmark = pytest.mark.gpu


def _quant_gpu(x_t, B=0, col_scale=None, flags=0, ldq_pad=0):
    rows, cols = x_t.shape
    q_full = torch.empty((rows, cols + ldq_pad), dtype=torch.int8, device="cuda")
    q = q_full[:, :cols]
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_quantize_rows(x_t, q, s, st, col_scale=col_scale, hadamard_block=B, flags=flags)
    return host(q), host(s), status_word(st)


CASES = [
    # rows, cols, B, dtype
    (32, 256, 256, torch.float32),     # tiny layer input
    (128, 256, 256, torch.float32),    # tiny layer weight prep
    (17, 5376, 128, torch.bfloat16),   # the 5376-wide layer, edge row count
    (1, 5376, 128, torch.bfloat16),
    (300, 144, 16, torch.bfloat16),    # chunk tail (144 = 256 - 112)
    (77, 400, 0, torch.float32),
    (64, 1040, 8, torch.float32),
    (9, 20480, 256, torch.bfloat16),   # long rows: two-pass kernel
    (5, 16384, 64, torch.float32),
    (3, 16, 2, torch.float32),
    (2, 4096, 4, torch.bfloat16),
    # >= 2 rows per SM and 9..32 chunks: rows staged by the bulk-copy engine
    (400, 2320, 16, torch.float32),    # 10 chunks, ragged last chunk
    (500, 5376, 128, torch.bfloat16),  # 21 chunks
    (320, 8192, 256, torch.bfloat16),  # 32 chunks
    (2000, 4096, 0, torch.float32),    # several rows per CTA through the ring
    # bf16, block 128, >= 4 rows per SM: 1024-column warps, pairs of rows per TMA load
    (1200, 5376, 128, torch.bfloat16),
    (601, 1024, 128, torch.bfloat16),  # odd row count: the last pair is half empty
    (700, 8192, 128, torch.bfloat16),
    (900, 2176, 128, torch.bfloat16),  # 2176 = 2 * 1024 + 128: a warp with one active block
]


@pytest.mark.parametrize("rows,cols,B,dtype", CASES)
def test_quantize_rows_bit_exact(rows, cols, B, dtype):
    x = workloads.normal((rows, cols), 1.0, rows * 7 + cols)
    x[:, : max(1, cols // 64)] *= np.float32(25.0)
    xt = torch.from_numpy(x).to(dtype)
    x32 = xt.float().numpy()
    q, s, st = _quant_gpu(dev(xt), B)
    rq, rs, rst = oracle.quantize_rows(x32, B=B)
    assert st == 0 and rst == 0
    assert np.array_equal(s, rs)
    assert np.array_equal(q, rq)


# bf16 rows that take the two-threads-per-block quantizer (at least one
# tile of R = min(32, 128 / blocks) rows per SM): every block width it
# instantiates, one 128-column block per row (R = 32) up to 128 blocks per row
# (R = 1), and row counts that leave a ragged last tile.
BLK_CASES = [
    # rows, cols, B
    (2400, 1024, 0), (2401, 1024, 2), (2400, 1024, 4), (2401, 1024, 8),
    (2400, 1024, 16), (2401, 1024, 32), (2400, 1024, 64), (2401, 1024, 128),
    (4801, 128, 128), (4801, 128, 64),
    (300, 16384, 128), (301, 16384, 32),
    (1337, 3456, 128),
]


@pytest.mark.parametrize("rows,cols,B", BLK_CASES)
def test_quantize_rows_block_quantizer_bit_exact(rows, cols, B):
    x = workloads.normal((rows, cols), 1.0, rows * 13 + cols + B)
    x[:, : max(1, cols // 64)] *= np.float32(25.0)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    x32 = xt.float().numpy()
    q, s, st = _quant_gpu(dev(xt), B)
    rq, rs, rst = oracle.quantize_rows(x32, B=B)
    assert st == 0 and rst == 0
    assert np.array_equal(s, rs)
    assert np.array_equal(q, rq)


@pytest.mark.parametrize("rows", [96, 700])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_rows_with_col_scale(dtype, rows):
    """The row quantization of dY * s_w that precedes the input-gradient GEMM."""
    x = workloads.normal((rows, 7168), 1.0, 3)
    cs = np.abs(workloads.normal((7168,), 1e-3, 4)) + np.float32(1e-5)
    xt = torch.from_numpy(x).to(dtype)
    q, s, st = _quant_gpu(dev(xt), 0, col_scale=dev(cs))
    rq, rs, rst = oracle.quantize_rows(xt.float().numpy(), col_scale=cs)
    assert st == rst == 0
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


def test_quantize_rows_strided_output_and_input():
    x = workloads.normal((40, 512), 1.0, 5)
    big = torch.zeros((40, 768), dtype=torch.float32)
    big[:, :512] = torch.from_numpy(x)
    xv = dev(big)[:, :512]
    q, s, st = _quant_gpu(xv, 128, ldq_pad=48)
    rq, rs, _ = oracle.quantize_rows(x, B=128)
    assert st == 0 and np.array_equal(q, rq) and np.array_equal(s, rs)


def test_quantize_zero_rows_and_nonfinite_flags():
    x = workloads.normal((8, 256), 1.0, 6)
    x[3] = 0.0
    q, s, st = _quant_gpu(dev(x), 0)
    assert st == 0 and s[3] == 0 and not q[3].any()
    q, s, st = _quant_gpu(dev(x), 16, flags=ql.QL_REJECT_ZERO_ROWS)
    assert st == (1 << ql.QL_ERR_ZERO_ROW)
    rq, rs, _ = oracle.quantize_rows(x, B=16, flags=oracle.REJECT_ZERO_ROWS)
    assert np.array_equal(q, rq) and np.array_equal(s, rs)
    x[5, 100] = np.nan
    _, _, st = _quant_gpu(dev(x), 0)
    assert st & (1 << ql.QL_ERR_NONFINITE)
    x[5, 100] = np.inf
    _, _, st = _quant_gpu(dev(x), 32)
    assert st & (1 << ql.QL_ERR_NONFINITE)


@pytest.mark.parametrize("B", [2, 8, 32, 128, 256])
@pytest.mark.parametrize("xt,yt", [(torch.float32, torch.float32),
                                   (torch.float32, torch.bfloat16),
                                   (torch.bfloat16, torch.float32),
                                   (torch.bfloat16, torch.bfloat16)])
def test_hadamard_matches_oracle(B, xt, yt):
    x = torch.from_numpy(workloads.normal((37, 768), 1.0, B)).to(xt)
    y = torch.empty((37, 768), dtype=yt, device="cuda")
    ql.qlinear_hadamard(dev(x), y, B)
    ref, st = oracle.hadamard_rows(x.float().numpy(), B)
    assert st == 0
    ref_t = torch.from_numpy(ref).to(yt).float().numpy()
    assert np.array_equal(host(y), ref_t)


def test_hadamard_in_place_twice_is_identity():
    x = workloads.normal((64, 5376), 1.0, 9)
    t = dev(x)
    ql.qlinear_hadamard(t, t, 128)
    ref, _ = oracle.hadamard_rows(x, 128)
    assert np.array_equal(host(t), ref)
    ql.qlinear_hadamard(t, t, 128)
    assert np.abs(host(t) - x).max() <= 1e-5 * np.abs(x).max()


def test_host_validation_errors():
    x = torch.zeros((4, 40), device="cuda")
    q = torch.zeros((4, 48), dtype=torch.int8, device="cuda")
    s = torch.zeros(4, device="cuda")
    st = new_status()
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_quantize_rows(x, q[:, :40], s, st)  # cols % 16 != 0
    assert e.value.code == ql.QL_ERR_SHAPE
    x = torch.zeros((4, 48), device="cuda")
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_quantize_rows(x, q, s, st, hadamard_block=3)
    assert e.value.code == ql.QL_ERR_ARG
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_quantize_rows(x, q, s, st, hadamard_block=32)  # 48 % 32 != 0
    assert e.value.code == ql.QL_ERR_SHAPE
    flat = torch.zeros(4 * 48 + 4, device="cuda")
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_quantize_rows(flat[1:1 + 4 * 48].view(4, 48), q, s, st)  # misaligned
    assert e.value.code == ql.QL_ERR_ALIGN
    assert status_word(st) == 0


@pytest.mark.parametrize("B", [0, 2, 16, 128, 256])
@pytest.mark.parametrize("wt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,K", [(37, 768), (300, 5376), (5, 16)])
def test_dequantize_matches_oracle(N, K, B, wt):
    """(s_w q) R back to the original basis: the same float32 operations in
    the same order as the oracle (bf16 output = the oracle's value rounded)."""
    if B and K % B:
        pytest.skip("block does not divide K")
    w = workloads.normal((N, K), 0.02, N + K + B)
    q, s, st = oracle.quantize_rows(w, B=B, flags=oracle.REJECT_ZERO_ROWS)
    assert st == 0
    out = torch.empty((N, K), dtype=wt, device="cuda")
    ql.qlinear_dequantize(dev(q), dev(s), B, out)
    ref, rst = oracle.dequantize(q, s, B)
    assert rst == 0
    ref_t = torch.from_numpy(ref).to(wt).float().numpy()
    assert np.array_equal(host(out), ref_t)


def test_dequantize_strided_output():
    q = np.random.Generator(np.random.PCG64(5)).integers(-127, 128, (24, 512)).astype(np.int8)
    s = workloads.uniform((24,), 1e-3, 1e-2, 6)
    big = torch.zeros((24, 640), device="cuda")
    ql.qlinear_dequantize(dev(q), dev(s), 64, big[:, :512])
    ref, _ = oracle.dequantize(q, s, 64)
    assert np.array_equal(host(big[:, :512]), ref) and not host(big[:, 512:]).any()
