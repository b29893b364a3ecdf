"""qlinear_bwd_dx_noalloc: the input gradient for callers that cannot
allocate device memory (for example code running inside a host framework
that owns all device memory and forbids allocation while it executes), so
cannot hand the library a workspace.  The entry point uses the library's
own fixed scratch array instead.

Checked through the C ABI on a GPU: two calls in a row, each against
qlinear_bwd_dx given a separately allocated workspace.  Both run the same
kernels on the same inputs, so the results must be identical bit for bit (a
tolerance could hide stale scratch contents leaking into an element); sizes
beyond the scratch capacity are rejected before anything runs.  This file sorts last so that a run that stops
at the first failure has already run every other test; it also passes alone
in a fresh process (its first call then does the one-time set-up)."""
from __future__ import annotations

import pytest
import torch

import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, new_status, status_word

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, B, dyt, seed):
    w = workloads.normal((N, K), 0.02, seed)
    dy = torch.from_numpy(workloads.normal((M, N), 1.0, seed + 1)).to(dyt)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    st = new_status()
    ql.qlinear_quantize_rows(dev(w), wq, sw, st, hadamard_block=B, flags=ql.QL_REJECT_ZERO_ROWS)
    assert status_word(st) == 0
    return dev(dy), wq, sw


def _with_workspace(dy, wq, sw, B, dxt):
    M, N = dy.shape
    K = wq.shape[1]
    # a workspace full of garbage: the call must not depend on its contents
    ws = torch.full((ql.qlinear_workspace_bytes(M, N, K, B),), 0xA5, dtype=torch.uint8,
                    device="cuda")
    dx = torch.empty((M, K), dtype=dxt, device="cuda")
    st = new_status()
    ql.qlinear_bwd_dx(dy, wq, sw, B, dx, ws, st)
    assert status_word(st) == 0
    return dx


CALLS = [
    # M, N, K, block, dy dtype, dx dtype: the fused block-128 rotation, then the
    # block-256 path whose float32 product also lives in the scratch array
    (300, 272, 384, 128, torch.bfloat16, torch.bfloat16),
    (64, 512, 256, 256, torch.float32, torch.bfloat16),
]


def test_noalloc_matches_workspace_call_twice_in_a_row():
    # each size twice, interleaved, so every call follows one that left other
    # contents in the scratch
    for i, (M, N, K, B, dyt, dxt) in enumerate(CALLS + CALLS):
        dy, wq, sw = _inputs(M, N, K, B, dyt, 500 + i)
        ref = _with_workspace(dy, wq, sw, B, dxt)
        dx = torch.empty((M, K), dtype=dxt, device="cuda")
        st = new_status()
        ql.qlinear_bwd_dx_noalloc(dy, wq, sw, B, dx, st)
        assert status_word(st) == 0
        # the scratch keeps the previous call's contents; the result must not
        # depend on them
        assert torch.equal(dx, ref), f"call {i}: differs from the workspace call"


def test_noalloc_rejects_sizes_beyond_the_scratch():
    M, N, K = 12000, 7168, 256
    assert ql.qlinear_workspace_bytes(M, N, K, 0) > ql.QL_NOALLOC_SCRATCH_BYTES
    dy = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sw = torch.ones(N, device="cuda")
    dx = torch.full((M, K), 3.0, device="cuda")
    st = new_status()
    with pytest.raises(ql.QLError) as e:
        ql.qlinear_bwd_dx_noalloc(dy, wq, sw, 0, dx, st)
    assert e.value.code == ql.QL_ERR_UNSUPPORTED
    assert bool((dx == 3.0).all()) and status_word(st) == 0
