"""Failure detection on the GPU, without a fault: every pipeline wait in the
library is bounded.  A test kernel waits, through the same bounded mbarrier
wait the GEMM and streaming kernels use, on a barrier that nothing ever
completes; the wait runs out, the kernel reports QL_ERR_TIMEOUT in the
status word and returns, and the CUDA context stays usable for the next
call (which must still be bit-exact against the oracle)."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, host, new_status, status_word

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_us", [1000, 50000])
def test_bounded_wait_reports_timeout_and_returns(limit_us):
    st = new_status()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ql.ql_test_wait_timeout(st, limit_us)
    word = status_word(st)
    elapsed = time.perf_counter() - t0
    assert word == 1 << ql.QL_ERR_TIMEOUT
    assert ql.status_flags(word) == ["TIMEOUT"]
    assert elapsed >= limit_us * 1e-6
    assert elapsed < limit_us * 1e-6 + 5.0


def test_context_usable_after_timeout():
    st = new_status()
    ql.ql_test_wait_timeout(st, 2000)
    assert status_word(st) == 1 << ql.QL_ERR_TIMEOUT
    x = workloads.normal((300, 5376), 1.0, 11)
    q = torch.empty((300, 5376), dtype=torch.int8, device="cuda")
    s = torch.empty(300, dtype=torch.float32, device="cuda")
    st2 = new_status()
    ql.qlinear_quantize_rows(dev(x), q, s, st2, hadamard_block=128)
    rq, rs, rst = oracle.quantize_rows(x, B=128)
    assert status_word(st2) == 0 and rst == 0
    assert np.array_equal(host(q), rq) and np.array_equal(host(s), rs)


def test_timeout_hook_argument_errors():
    st = new_status()
    with pytest.raises(ql.QLError) as e:
        ql.ql_test_wait_timeout(st, 0)
    assert e.value.code == ql.QL_ERR_ARG
    assert status_word(st) == 0
