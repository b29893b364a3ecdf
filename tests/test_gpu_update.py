"""GPU parity of the fused optimizer step + stochastic requantization against
the oracle, through the C ABI.  New codes, scales, moments and (for weight
norm) magnitudes must be bit-exact: both sides evaluate the same float32
operations in the same order and draw the same Philox4x32-10 words."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, host, new_status, status_word

pytestmark = pytest.mark.gpu


def prepared(d):
    q, s, st = oracle.quantize_rows(d["w"], flags=oracle.REJECT_ZERO_ROWS)
    assert st == 0
    return q, s


def run_gpu(q, s, grad, kind, lr, seed, step, m=None, v=None, wd=0.0, g=None, g_m=None,
            g_v=None):
    tq, ts, tg = dev(q), dev(s), dev(grad)
    tm = dev(m) if m is not None else None
    tv = dev(v) if v is not None else None
    tgm = [dev(a) if a is not None else None for a in (g, g_m, g_v)]
    st = new_status()
    opt = ql.Optim(kind=kind, lr=lr, weight_decay=wd)
    ql.qweight_update_sr(tq, ts, tg, opt, tm, tv, seed, step, st, g=tgm[0], g_m=tgm[1], g_v=tgm[2])
    word = status_word(st)
    out = [host(tq), host(ts), host(tm) if tm is not None else None,
           host(tv) if tv is not None else None] + [host(a) if a is not None else None for a in tgm]
    return out, word


def check_equal(gpu, ref, names):
    for a, b, n in zip(gpu, ref, names):
        if b is None:
            continue
        assert a.shape == b.shape, n
        bad = a.view(np.uint8) != b.view(np.uint8) if a.dtype != np.int8 else a != b
        assert not bad.any(), f"{n}: {int(bad.sum())} elements differ"


NAMES = ["codes", "scales", "m", "v", "g", "g_m", "g_v"]


@pytest.mark.parametrize("N,K", [(128, 256), (64, 1024), (33, 5376), (16, 16384), (8, 32768),
                                 (40, 400), (5, 16)])
def test_sgd_update_bit_exact(N, K):
    d = workloads.update_state(N, K, seed=N)
    q, s = prepared(d)
    gpu, st = run_gpu(q, s, d["grad"], ql.QL_SGD, 1e-2, seed=0, step=1)
    ref = oracle.update_sr(q, s, d["grad"], oracle.SGD, 1e-2, seed=0, step=1)
    assert st == 0 and ref[-1] == 0
    check_equal(gpu[:2], ref[:2], NAMES)


@pytest.mark.parametrize("warm", [False, True])
# Rows up to ~8K elements are staged in shared memory; longer ones
# (14336, 16384, 32768, 14352: a 16-element last piece) stream through the
# piece ring, each CTA one row here and several rows in the sampled full sizes.
@pytest.mark.parametrize("N,K", [(64, 1024), (48, 4096), (24, 14336), (16, 16384), (100, 272),
                                 (6, 32768), (5, 14352)])
def test_adamw_update_bit_exact(N, K, warm):
    d = workloads.update_state(N, K, seed=K + warm, warm=warm)
    q, s = prepared(d)
    seed = 0x1234_5678_9ABC
    gpu, st = run_gpu(q, s, d["grad"], ql.QL_ADAMW, 1e-3, seed, d["step"], m=d["m"], v=d["v"],
                      wd=0.01)
    ref = oracle.update_sr(q, s, d["grad"], oracle.ADAMW, 1e-3, seed, d["step"], m=d["m"],
                           v=d["v"], wd=0.01)
    assert st == 0 and ref[-1] == 0
    check_equal(gpu[:4], ref[:4], NAMES)


@pytest.mark.parametrize("kind", [ql.QL_ADAMW, ql.QL_SGD])
# Weight-norm rows of every length stage their codes and gradient, one row
# per CTA: K = 80 with fewer groups than lanes, K = 18448 and 32768 with
# two and one rows per SM.
# AdamW rows up to K = 5584 stage their moments too (352 threads there,
# more than the 256 virtual lanes); K = 5600 is the first that does not.
# Streamed moments are loaded one chunk ahead up to K = 10640, four chunks
# ahead from K = 10656 on.
@pytest.mark.parametrize("N,K", [(32, 1024), (12, 4096), (6, 16384), (20, 80), (160, 18448),
                                 (4, 32768), (10, 5584), (10, 5600), (6, 10640), (6, 10656)])
def test_weight_norm_update_bit_exact(N, K, kind):
    d = workloads.update_state(N, K, seed=3 * K, weight_norm=True)
    q, s = prepared(d)
    adam = kind == ql.QL_ADAMW
    kw = dict(m=d["m"], v=d["v"], wd=0.01) if adam else {}
    gpu, st = run_gpu(q, s, d["grad"], kind, 1e-3, 99, 1, g=d["g"],
                      g_m=d["g_m"] if adam else None, g_v=d["g_v"] if adam else None, **kw)
    ref = oracle.update_sr(q, s, d["grad"], kind, 1e-3, 99, 1, g=d["g"],
                           g_m=d["g_m"] if adam else None, g_v=d["g_v"] if adam else None, **kw)
    assert st == 0 and ref[-1] == 0
    check_equal(gpu, ref[:7], NAMES)


# Zero directions among other rows, in each form of the weight-norm kernel:
# K = 512 (moments staged), 6160 (one chunk of moments ahead), 18448 and
# 32768 (four chunks ahead; two and one rows per SM)
@pytest.mark.parametrize("N,K,zero", [(6, 512, [2]), (300, 6160, [0, 2, 149, 299]),
                                      (300, 18448, [0, 2, 149, 299]), (160, 32768, [3, 150])])
def test_weight_norm_zero_direction_flagged_and_untouched(N, K, zero):
    d = workloads.update_state(N, K, seed=5, weight_norm=True, warm=True)
    q, s = prepared(d)
    q[zero] = 0
    s[zero] = 0
    gpu, st = run_gpu(q, s, d["grad"], ql.QL_ADAMW, 1e-3, 1, d["step"], m=d["m"], v=d["v"],
                      g=d["g"], g_m=d["g_m"], g_v=d["g_v"])
    ref = oracle.update_sr(q, s, d["grad"], oracle.ADAMW, 1e-3, 1, d["step"], m=d["m"], v=d["v"],
                           g=d["g"], g_m=d["g_m"], g_v=d["g_v"])
    assert st == (1 << ql.QL_ERR_ZERO_ROW) and ref[-1] == oracle.BIT_ZERO_ROW
    check_equal(gpu, ref[:7], NAMES)


SAMPLED = [
    # N, K, warm moments, weight norm
    (1024, 1024, True, False),      # the [1024,1024] .. [16384,16384] sweep
    (2048, 2048, False, True),
    (4096, 4096, False, False),
    (8192, 8192, True, False),
    (8192, 8192, False, True),
    (16384, 16384, False, False),
    (16384, 16384, False, True),
    (14336, 4096, True, False),     # SwiGLU w1 / w3
    (28672, 4096, True, False),     # w1 and w3 stacked
    (4096, 14336, True, False),     # SwiGLU w2
]


@pytest.mark.slow
@pytest.mark.parametrize("N,K,warm,wn", SAMPLED)
def test_adamw_full_size_sampled_rows(N, K, warm, wn):
    """Full-size AdamW updates (plain and row-wise weight norm): the whole
    matrix updates on the GPU; sampled rows are recomputed by the oracle,
    whose random stream is keyed by the absolute row."""
    d = workloads.update_state(N, K, seed=N + K, warm=warm, weight_norm=wn)
    q0, s0 = prepared(d)
    del d["w"]
    tq, ts, tg = dev(q0), dev(s0), dev(d["grad"])
    if warm:
        tm, tv = dev(d["m"]), dev(d["v"])
    else:
        tm = torch.zeros((N, K), device="cuda")
        tv = torch.zeros((N, K), device="cuda")
    wn_t = [dev(d[k]) for k in ("g", "g_m", "g_v")] if wn else [None] * 3
    seed = 0xC0FFEE + N
    st = new_status()
    ql.qweight_update_sr(tq, ts, tg, ql.Optim(weight_decay=0.01), tm, tv, seed, d["step"], st,
                         g=wn_t[0], g_m=wn_t[1], g_v=wn_t[2])
    assert status_word(st) == 0
    del tg
    rows = np.array(sorted({0, 1, N // 2, N - 1} | set(
        np.random.Generator(np.random.PCG64(N * 3 + K)).integers(0, N, 10).tolist())))
    ri = torch.from_numpy(rows).cuda()
    got = [host(tq[ri]), host(ts[ri]), host(tm[ri]), host(tv[ri])]
    got += [host(t[ri]) for t in wn_t] if wn else [None] * 3
    for i, r in enumerate(rows):
        r = int(r)
        sl = slice(r, r + 1)
        kw = dict(g=d["g"][sl], g_m=d["g_m"][sl], g_v=d["g_v"][sl]) if wn else {}
        ref = oracle.update_sr(q0[sl], s0[sl], d["grad"][sl], oracle.ADAMW, 1e-3, seed,
                               d["step"], m=d["m"][sl], v=d["v"][sl], wd=0.01, row0=r, **kw)
        assert ref[-1] == 0
        check_equal([None if a is None else a[i:i + 1] for a in got], ref[:7], NAMES)


def test_update_argument_errors():
    q = torch.zeros((4, 32), dtype=torch.int8, device="cuda")
    s = torch.ones(4, device="cuda")
    g = torch.zeros((4, 32), device="cuda")
    st = new_status()
    with pytest.raises(ql.QLError) as e:
        ql.qweight_update_sr(q, s, g, ql.Optim(kind=ql.QL_SGD, weight_decay=0.1), None, None, 0, 1, st)
    assert e.value.code == ql.QL_ERR_ARG
    with pytest.raises(ql.QLError) as e:
        ql.qweight_update_sr(q, s, g, ql.Optim(kind=ql.QL_SGD, weight_decay=0.0), None, None, 0, 0, st)
    assert e.value.code == ql.QL_ERR_ARG
    with pytest.raises(ql.QLError) as e:
        ql.qweight_update_sr(q, s, g, ql.Optim(), None, None, 0, 1, st)  # AdamW needs m, v
    assert e.value.code == ql.QL_ERR_ARG
    assert status_word(st) == 0
