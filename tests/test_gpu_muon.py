"""GPU parity of MuonAuxAdamW against the oracle, through the C ABI.

Staged, as every update path of the layer: the momentum is bit for bit; the
orthogonalized update O runs Newton-Schulz with bf16 operands (as the
published method does) and is compared with the oracle's float64 iteration
of the same definition within a bound of bf16 accuracy, and by the property
the quintic iteration guarantees (every singular value of O inside its band);
the Muon requantization step is bit for bit given the GPU's own O; the AdamW
on float vectors is bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, host, new_status, status_word

pytestmark = pytest.mark.gpu

# Relative Frobenius distance of the bf16 Newton-Schulz result from the
# float64 one: bf16 keeps 8 significant bits (relative rounding 2^-9 ~ 2e-3
# per stored value); each step stores X, A and B once, five steps, and the
# iteration contracts errors toward its fixed band rather than amplifying
# them, so a few percent bounds it.
NS_REL_TOL = 3e-2


def _orthogonalize(G, M, beta=0.95, steps=5):
    N, K = G.shape
    g, m = dev(G), dev(M)
    O = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ql.qweight_muon_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    st = new_status()
    ql.qweight_muon_orthogonalize(g, m, O, ws, st, momentum=beta, ns_steps=steps)
    assert status_word(st) == 0
    return host(m), O


@pytest.mark.parametrize("N,K", [(256, 384), (384, 256), (128, 128), (16, 1040),
                                 # two 256-tiles a side with a ragged second one: the
                                 # symmetric products' upper-tile path and its mirror
                                 (400, 640), (640, 400), (784, 784)])
def test_momentum_bit_exact_and_newton_schulz_close(N, K):
    G = workloads.normal((N, K), 1e-3, N + K)
    M = workloads.normal((N, K), 1e-3, N + K + 1)
    m_gpu, O = _orthogonalize(G, M)
    rM, rU = oracle.muon_momentum(G, M, 0.95)
    assert np.array_equal(m_gpu, rM)
    ref = oracle.newton_schulz5(rU)
    o = host(O).astype(np.float64)
    assert np.linalg.norm(o - ref) <= NS_REL_TOL * np.linalg.norm(ref)
    # the iteration acts on singular values: the GPU's track the float64 ones
    # (a square U has singular values near 0 that five steps leave below the
    # band, on both sides)
    sv, sv_ref = (np.linalg.svd(a, compute_uv=False) for a in (o, ref))
    assert np.abs(sv - sv_ref).max() <= 0.05 and sv.max() < 1.3


@pytest.mark.parametrize("N,K", [(256, 384), (384, 256)])
def test_muon_step_bit_exact_given_O(N, K):
    d = workloads.update_state(N, K, seed=N * 3 + K)
    q, s, st = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    assert st == 0
    _, O = _orthogonalize(d["grad"], np.zeros((N, K), np.float32))
    o32 = host(O)  # the GPU's own bf16 update, exact in float32
    tq, ts = dev(q), dev(s)
    stw = new_status()
    ql.qweight_update_muon_sr(tq, ts, O, 0.02, 0.01, seed=77, step=4, status=stw)
    assert status_word(stw) == 0
    rq, rs, rst = oracle.update_muon_sr(q, s, o32, 0.02, 0.01, seed=77, step=4)
    assert rst == 0
    assert np.array_equal(host(ts), rs) and np.array_equal(host(tq), rq)


@pytest.mark.parametrize("n", [1, 300, 7168])
def test_vector_adamw_bit_exact(n):
    p = workloads.normal((n,), 0.01, n)
    g = workloads.normal((n,), 1e-3, n + 1)
    m = workloads.normal((n,), 1e-4, n + 2)
    v = np.square(workloads.normal((n,), 1e-3, n + 3))
    tp, tm, tv = dev(p), dev(m), dev(v)
    st = new_status()
    ql.qvector_adamw(tp, dev(g), tm, tv, ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.01),
                     10, st)
    assert status_word(st) == 0
    rp, rm, rv, rst = oracle.adamw_vector(p, g, m, v, 1e-3, step=10, wd=0.01)
    assert rst == 0
    assert np.array_equal(host(tp), rp) and np.array_equal(host(tm), rm)
    assert np.array_equal(host(tv), rv)


def test_full_layer_weight_properties_and_sampled_rows():
    """The 5376 -> 7168 layer's weight (N = 7168 > K = 5376: the iteration
    runs on U^T): momentum bit for bit in full; O's squared Frobenius norm per
    singular value and its largest singular value (power iteration) inside the
    iteration's band; the requantization bit for bit on sampled rows."""
    N, K = 7168, 5376
    d = workloads.update_state(N, K, seed=3, warm=True)
    q, s, _ = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    m_gpu, O = _orthogonalize(d["grad"], d["m"])
    rM, _ = oracle.muon_momentum(d["grad"], d["m"], 0.95)
    assert np.array_equal(m_gpu, rM)
    Of = O.float()
    fro2 = float((Of * Of).sum()) / min(N, K)
    assert 0.3 < fro2 < 1.3
    x = torch.randn(K, device="cuda", generator=torch.Generator(device="cuda").manual_seed(0))
    for _ in range(30):
        x = Of.T @ (Of @ x)
        x = x / x.norm()
    smax = float((Of @ x).norm())
    assert smax < 1.3
    tq, ts = dev(q), dev(s)
    st = new_status()
    ql.qweight_update_muon_sr(tq, ts, O, 0.02, 0.01, seed=5, step=9, status=st)
    assert status_word(st) == 0
    rows = [0, 1, 127, 128, 4000, N - 1]
    o32 = host(O)
    q_gpu, s_gpu = host(tq), host(ts)
    for r in rows:  # each sampled row keyed by its own index in the weight
        q1, s1, st1 = oracle.update_muon_sr(q[r:r + 1], s[r:r + 1], o32[r:r + 1], 0.02, 0.01,
                                            seed=5, step=9, n_full=N, row0=r)
        assert st1 == 0 and np.array_equal(q_gpu[r], q1[0]) and s_gpu[r] == s1[0]


def test_muon_validation():
    st = new_status()
    g = torch.zeros((32, 40), device="cuda")
    with pytest.raises(ql.QLError) as e:   # K % 16 != 0
        ql.qweight_muon_orthogonalize(g, torch.zeros_like(g),
                                      torch.zeros((32, 40), dtype=torch.bfloat16, device="cuda"),
                                      torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), st)
    assert e.value.code == ql.QL_ERR_SHAPE
    g = torch.zeros((32, 48), device="cuda")
    with pytest.raises(ql.QLError) as e:   # ns_steps out of range
        ql.qweight_muon_orthogonalize(g, torch.zeros_like(g),
                                      torch.zeros((32, 48), dtype=torch.bfloat16, device="cuda"),
                                      torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), st,
                                      ns_steps=0)
    assert e.value.code == ql.QL_ERR_ARG
    assert status_word(st) == 0
