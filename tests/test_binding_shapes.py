"""The Python binding's operand-size checks, on the CPU.

The C ABI receives plain pointers, so a tensor that is too short for the
sizes passed with it can only be refused by the binding.  These tests stub
the library and the device pointers: every call pattern used by the GPU
tests, the benchmark and smoke() (including the empty and degenerate sizes)
must pass the checks, and each undersized or mis-shaped operand must raise
ValueError before any library call.
"""
from __future__ import annotations

import pytest
import torch

import int8_quantized_act_b200 as ql


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append(name)
            return 0
        return f


@pytest.fixture
def fake(monkeypatch):
    L = _FakeLib()
    monkeypatch.setattr(ql, "lib", lambda: L)
    monkeypatch.setattr(ql, "_dev", lambda t, what, dtype=None: None if t is None else 16)
    monkeypatch.setattr(ql, "_stream", lambda s: None)
    return L


def E(*shape, dtype=torch.float32):
    return torch.empty(shape, dtype=dtype)


I8, BF = torch.int8, torch.bfloat16
M, K, N = 32, 256, 128


def st():
    return E(1, dtype=torch.int32)


# ------------------------------------------------------------------ accepted
def test_valid_calls_pass(fake):
    ql.qlinear_quantize_rows(E(4, 48), E(4, 48, dtype=I8), E(4), st())
    ql.qlinear_quantize_rows(E(4, 40), E(4, 48, dtype=I8)[:, :40], E(4), st())
    ql.qlinear_quantize_rows(E(4, 48), E(4, 64, dtype=I8)[:, :48], E(4), st(), col_scale=E(48))
    ql.qlinear_quantize_rows(E(0, 48), E(0, 48, dtype=I8), E(0), st())
    ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N), E(N), 128, E(M, N), E(M, K, dtype=I8),
                   E(M), st())
    ql.qlinear_fwd(E(1, K), E(N, K, dtype=I8), E(N), None, 128, E(1, N), E(1, K, dtype=I8),
                   E(1), st())
    # the SwiGLU gate, its backward and the forward from codes (the MLP step)
    ql.qlinear_swiglu_quantize(E(M, 2 * K, dtype=BF), E(M, K, dtype=I8), E(M), st())
    ql.qlinear_swiglu_bwd(E(M, 2 * K, dtype=BF), E(M, K, dtype=BF), E(M, 2 * K, dtype=BF))
    ql.qlinear_swiglu_bwd(E(M, 2 * K), E(M, K), E(M, 2 * K))
    ql.qlinear_fwd_quantized(E(M, K, dtype=I8), E(M), E(N, K, dtype=I8), E(N), E(N), E(M, N), st())
    # MuonAuxAdamW (the Muon GPU tests and bench)
    ql.qweight_muon_orthogonalize(E(M, K), E(M, K), E(M, K, dtype=BF),
                                  E(ql.qweight_muon_workspace_bytes(M, K), dtype=torch.uint8), st())
    ql.qweight_update_muon_sr(E(M, K, dtype=I8), E(M), E(M, K, dtype=BF), 0.02, 0.01, 1, 1, st())
    ql.qvector_adamw(E(N), E(N), E(N), E(N), ql.Optim(), 1, st())
    # M = 0 and K = 0 (the degenerate-size GPU test)
    ql.qlinear_fwd(E(0, 64), E(32, 64, dtype=I8), E(32), None, 0, E(0, 32), E(0, 64, dtype=I8),
                   E(0), st())
    ql.qlinear_fwd(E(5, 0), E(32, 0, dtype=I8), E(32), E(32), 0, E(5, 32), E(5, 0, dtype=I8),
                   E(5), st())
    ql.qlinear_fwd_bf16(E(M, K), E(N, K, dtype=BF), E(N), E(N), 128, E(M, N), E(64, dtype=torch.uint8),
                        st())
    ql.qlinear_fwd_bf16(E(5, 0, dtype=BF), E(32, 0, dtype=BF), E(32), E(32), 0, E(5, 32), None, st())
    ws = E(64, dtype=torch.uint8)
    ql.qlinear_bwd_dx(E(M, N), E(N, K, dtype=I8), E(N), 128, E(M, K), ws, st())
    ql.qlinear_bwd_dx_noalloc(E(M, N, dtype=BF), E(N, K, dtype=I8), E(N), 128, E(M, K, dtype=BF), st())
    ql.qlinear_bwd_dw(E(M, N), E(M, K, dtype=I8), E(M), E(N, K), E(N), ws, st())
    ql.qlinear_bwd_dw(E(M, N), E(M, K, dtype=I8), E(M), E(N, K), None, ws, st())
    ql.qlinear_bwd_dw(E(0, 32), E(0, 64, dtype=I8), E(0), E(32, 64), E(32), ws, st())
    ql.qlinear_bwd(E(M, N), E(N, K, dtype=I8), E(N), E(M, K, dtype=I8), E(M), 128, E(M, K),
                   E(N, K), E(N), ws, st())
    ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K), ql.Optim(kind=ql.QL_SGD, weight_decay=0.0),
                         None, None, 0, 1, st())
    ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K), ql.Optim(), E(N, K), E(N, K), 0, 1, st())
    ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K), ql.Optim(), E(N, K), E(N, K), 0, 1, st(),
                         g=E(N), g_m=E(N), g_v=E(N))
    ql.qlinear_dequantize(E(N, K, dtype=I8), E(N), 128, E(N, K))
    ql.qlinear_dequantize(E(24, 512, dtype=I8), E(24), 64, E(24, 640)[:, :512])
    assert len(fake.calls) == 30


# ------------------------------------------------------------------ refused
BAD = [
    ("quantize: q too narrow",
     lambda: ql.qlinear_quantize_rows(E(4, 48), E(4, 32, dtype=I8), E(4), st())),
    ("quantize: q too short",
     lambda: ql.qlinear_quantize_rows(E(4, 48), E(3, 48, dtype=I8), E(4), st())),
    ("quantize: row_scale short",
     lambda: ql.qlinear_quantize_rows(E(4, 48), E(4, 48, dtype=I8), E(3), st())),
    ("quantize: col_scale short",
     lambda: ql.qlinear_quantize_rows(E(4, 48), E(4, 48, dtype=I8), E(4), st(), col_scale=E(32))),
    ("quantize: no status word",
     lambda: ql.qlinear_quantize_rows(E(4, 48), E(4, 48, dtype=I8), E(4), E(0, dtype=torch.int32))),
    ("fwd: wq contraction differs",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K + 16, dtype=I8), E(N), None, 0, E(M, N),
                            E(M, K, dtype=I8), E(M), st())),
    ("fwd: y too small",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N), None, 0, E(M - 1, N),
                            E(M, K, dtype=I8), E(M), st())),
    ("fwd: sw short",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N - 1), None, 0, E(M, N),
                            E(M, K, dtype=I8), E(M), st())),
    ("fwd: bias short",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N), E(N - 1), 0, E(M, N),
                            E(M, K, dtype=I8), E(M), st())),
    ("fwd: saved codes of another width",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N), None, 0, E(M, N),
                            E(M, K - 16, dtype=I8), E(M), st())),
    ("fwd: saved scales short",
     lambda: ql.qlinear_fwd(E(M, K), E(N, K, dtype=I8), E(N), None, 0, E(M, N),
                            E(M, K, dtype=I8), E(M - 1), st())),
    ("fwd_bf16: y of another width",
     lambda: ql.qlinear_fwd_bf16(E(M, K), E(N, K, dtype=BF), E(N), None, 0, E(M, N + 1), None, st())),
    ("bwd_dx: weight has fewer rows than dY columns",
     lambda: ql.qlinear_bwd_dx(E(M, N), E(N - 1, K, dtype=I8), E(N), 0, E(M, K),
                               E(64, dtype=torch.uint8), st())),
    ("bwd_dx: dx too small",
     lambda: ql.qlinear_bwd_dx(E(M, N), E(N, K, dtype=I8), E(N), 0, E(M - 1, K),
                               E(64, dtype=torch.uint8), st())),
    ("bwd_dx_noalloc: sw short",
     lambda: ql.qlinear_bwd_dx_noalloc(E(M, N), E(N, K, dtype=I8), E(N - 1), 0, E(M, K), st())),
    ("bwd_dw: saved codes have fewer rows than dY",
     lambda: ql.qlinear_bwd_dw(E(M, N), E(M - 1, K, dtype=I8), E(M), E(N, K), None,
                               E(64, dtype=torch.uint8), st())),
    ("bwd_dw: dw of another width",
     lambda: ql.qlinear_bwd_dw(E(M, N), E(M, K, dtype=I8), E(M), E(N, K - 16), None,
                               E(64, dtype=torch.uint8), st())),
    ("bwd_dw: db short",
     lambda: ql.qlinear_bwd_dw(E(M, N), E(M, K, dtype=I8), E(M), E(N, K), E(N - 1),
                               E(64, dtype=torch.uint8), st())),
    ("bwd: saved scales short",
     lambda: ql.qlinear_bwd(E(M, N), E(N, K, dtype=I8), E(N), E(M, K, dtype=I8), E(M - 1), 0,
                            E(M, K), E(N, K), E(N), E(64, dtype=torch.uint8), st())),
    ("bwd: dw too small",
     lambda: ql.qlinear_bwd(E(M, N), E(N, K, dtype=I8), E(N), E(M, K, dtype=I8), E(M), 0,
                            E(M, K), E(N - 1, K), E(N), E(64, dtype=torch.uint8), st())),
    ("update: gradient of another width",
     lambda: ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K - 16), ql.Optim(), E(N, K),
                                  E(N, K), 0, 1, st())),
    ("update: moments too small",
     lambda: ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K), ql.Optim(), E(N - 1, K),
                                  E(N, K), 0, 1, st())),
    ("update: scales short",
     lambda: ql.qweight_update_sr(E(N, K, dtype=I8), E(N - 1), E(N, K), ql.Optim(), E(N, K),
                                  E(N, K), 0, 1, st())),
    ("update: magnitude short",
     lambda: ql.qweight_update_sr(E(N, K, dtype=I8), E(N), E(N, K), ql.Optim(), E(N, K),
                                  E(N, K), 0, 1, st(), g=E(N - 1), g_m=E(N), g_v=E(N))),
    ("dequantize: scales short",
     lambda: ql.qlinear_dequantize(E(N, K, dtype=I8), E(N - 1), 0, E(N, K))),
    ("fwd from codes: scales short",
     lambda: ql.qlinear_fwd_quantized(E(M, K, dtype=I8), E(M - 1), E(N, K, dtype=I8), E(N),
                                      None, E(M, N), st())),
    ("fwd from codes: y too small",
     lambda: ql.qlinear_fwd_quantized(E(M, K, dtype=I8), E(M), E(N, K, dtype=I8), E(N), None,
                                      E(M - 1, N), st())),
    ("muon: momentum too small",
     lambda: ql.qweight_muon_orthogonalize(E(M, K), E(M - 1, K), E(M, K, dtype=BF),
                                           E(1 << 22, dtype=torch.uint8), st())),
    ("muon step: update of another shape",
     lambda: ql.qweight_update_muon_sr(E(M, K, dtype=I8), E(M), E(M, K - 16, dtype=BF), 0.02, 0.0,
                                       1, 1, st())),
    ("vector adamw: moments short",
     lambda: ql.qvector_adamw(E(N), E(N), E(N - 1), E(N), ql.Optim(), 1, st())),
    ("gate: codes too narrow",
     lambda: ql.qlinear_swiglu_quantize(E(M, 2 * K, dtype=BF), E(M, K - 16, dtype=I8), E(M), st())),
    ("gate: scales short",
     lambda: ql.qlinear_swiglu_quantize(E(M, 2 * K, dtype=BF), E(M, K, dtype=I8), E(M - 1), st())),
    ("gate backward: dh too small",
     lambda: ql.qlinear_swiglu_bwd(E(M, 2 * K, dtype=BF), E(M - 1, K, dtype=BF), E(M, 2 * K, dtype=BF))),
    ("gate backward: output too small",
     lambda: ql.qlinear_swiglu_bwd(E(M, 2 * K, dtype=BF), E(M, K, dtype=BF), E(M, 2 * K - 16, dtype=BF))),
]


@pytest.mark.parametrize("name,call", BAD, ids=[b[0] for b in BAD])
def test_undersized_operands_are_refused(fake, name, call):
    with pytest.raises(ValueError):
        call()
    assert fake.calls == []  # refused before any library call
