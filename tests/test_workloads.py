"""The seeded input generators against the input recipe they state.

These pin what every parity test and the benchmark are fed: the shapes, the
distributions, the outlier channels of the rotated layer, the bf16 rounding
of the inputs, and the SwiGLU stage inputs (recomputed here in float64, with
the gating derivative checked by finite differences).  CPU only.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads


def _moments_ok(x: np.ndarray, std: float, k: float = 5.0) -> None:
    """Mean and standard deviation of a large N(0, std^2) sample, within k
    standard errors."""
    x = x.astype(np.float64).ravel()
    n = x.size
    assert abs(x.mean()) < k * std / np.sqrt(n)
    # standard error of the sample std of a normal sample: std / sqrt(2n)
    assert abs(x.std() - std) < k * std / np.sqrt(2 * n)


def test_draws_are_seeded_and_distinct():
    a = workloads.normal((64, 64), 1.0, 5)
    assert np.array_equal(a, workloads.normal((64, 64), 1.0, 5))
    assert not np.array_equal(a, workloads.normal((64, 64), 1.0, 6))
    assert a.dtype == np.float32


@pytest.mark.parametrize("std", [1.0, 0.02, 1e-3])
def test_normal_moments(std):
    _moments_ok(workloads.normal((400, 500), std, 1), std)


def test_uniform_range_and_mean():
    u = workloads.uniform((200_000,), 0.5, 2.0, 3).astype(np.float64)
    assert u.min() >= 0.5 and u.max() < 2.0
    # U(a, b): mean (a + b) / 2, standard deviation (b - a) / sqrt(12)
    assert abs(u.mean() - 1.25) < 5 * (1.5 / np.sqrt(12)) / np.sqrt(u.size)


def test_outlier_channels_of_the_rotated_layer():
    ch = workloads.outlier_channels(5376, 0.01, 0)
    assert ch.size == 54                      # round(0.01 * 5376)
    assert np.all(np.diff(ch) > 0) and ch[0] >= 0 and ch[-1] < 5376
    assert np.array_equal(ch, workloads.outlier_channels(5376, 0.01, 0))


def test_bf16_cast_rounds_to_nearest_even():
    one = np.float32(1.0)
    vals = np.array([one + np.float32(2.0**-8),        # halfway 1 | 1+2^-7: even is 1
                     one + np.float32(3 * 2.0**-8),    # halfway 1+2^-7 | 1+2^-6: even is 1+2^-6
                     one + np.float32(2.0**-8 + 2.0**-20),  # above halfway: up
                     np.float32(-3.0)], np.float32)
    t, x32 = workloads.to_bf16(vals)
    assert t.dtype == torch.bfloat16
    assert x32.tolist() == [1.0, 1.0 + 2.0**-6, 1.0 + 2.0**-7, -3.0]


def test_tiny_layer_recipe():
    d = workloads.tiny_layer(0)
    assert (d["M"], d["K"], d["N"], d["block"]) == (32, 256, 128, 256)
    raw = workloads.normal((32, 256), 1.0, 1)
    assert np.array_equal(d["x"][:, :4], raw[:, :4] * np.float32(20.0))
    assert np.array_equal(d["x"][:, 4:], raw[:, 4:])
    assert d["w"].shape == (128, 256) and d["bias"].shape == (128,)
    assert d["dy"].shape == (32, 128)
    assert d["lr"] == 1e-2 and d["step"] == 1


def test_rotated_layer_recipe():
    d = workloads.rotated_layer(M=256, seed=0)
    M, K, N = d["M"], d["K"], d["N"]
    assert (M, K, N, d["block"]) == (256, 5376, 7168, 128) and K % d["block"] == 0
    x = d["x"]
    # bf16 inputs: the float32 copy is exactly the bf16 tensor's value
    assert torch.equal(torch.from_numpy(x).to(torch.bfloat16), d["x_bf16"])
    assert np.array_equal(d["x_bf16"].float().numpy(), x)
    mask = np.zeros(K, bool)
    mask[d["outliers"]] = True
    assert mask.sum() == 54
    # outlier channels are the N(0,1) draw scaled x30 (then rounded to bf16)
    raw = workloads.normal((M, K), 1.0, 11)
    assert np.array_equal(x[:, mask], workloads.to_bf16(raw[:, mask] * np.float32(30.0))[1])
    assert np.array_equal(x[:, ~mask], workloads.to_bf16(raw[:, ~mask])[1])
    _moments_ok(x[:, ~mask], 1.0, k=6.0)
    _moments_ok(x[:, mask], 30.0, k=6.0)
    _moments_ok(d["w"], 0.02)
    assert d["dy_bf16"].shape == (M, N) and d["dy_bf16"].dtype == torch.bfloat16


def test_swiglu_mlp_shapes():
    d = workloads.swiglu_mlp(T=32, d_model=64, d_ff=96)
    assert d["x_bf16"].shape == (32, 64) and d["dy_bf16"].shape == (32, 64)
    assert d["w1"].shape == (96, 64) and d["w3"].shape == (96, 64)
    assert d["w2"].shape == (64, 96)
    assert d["lr"] == 1e-3


def test_swiglu_gate_inputs_recipe():
    T, F = 64, 512
    d = workloads.swiglu_gate_inputs(T=T, d_ff=F, seed=0)
    sd = 0.02 * 64.0
    assert d["ab"].shape == (T, 2 * F) and d["dh"].shape == (T, F)
    _moments_ok(d["ab"][:, :F], sd)
    _moments_ok(d["ab"][:, F:], sd)
    _moments_ok(d["dh"], sd)
    # a and b are independent draws, each the bf16 rounding of its float32 draw
    a = workloads.normal((T, F), sd, 41)
    b = workloads.normal((T, F), sd, 42)
    assert np.array_equal(d["ab"][:, :F], workloads.to_bf16(a)[1])
    assert np.array_equal(d["ab"][:, F:], workloads.to_bf16(b)[1])
    assert np.array_equal(d["ab_bf16"].float().numpy(), d["ab"])
    assert np.array_equal(d["dh_bf16"].float().numpy(), d["dh"])


@pytest.mark.parametrize("warm", [False, True])
def test_update_state_recipe(warm):
    d = workloads.update_state(64, 512, seed=0, warm=warm, weight_norm=True)
    assert d["step"] == (10 if warm else 1)
    _moments_ok(d["w"], 0.02)
    _moments_ok(d["grad"], 1e-3)
    if warm:
        _moments_ok(d["m"], 1e-4)
        v = d["v"].astype(np.float64)
        assert np.all(v >= 0)
        # v = z^2 with z ~ N(0, 1e-3^2): mean 1e-6, standard deviation sqrt(2) * 1e-6
        assert abs(v.mean() - 1e-6) < 5 * np.sqrt(2) * 1e-6 / np.sqrt(v.size)
    else:
        assert not d["m"].any() and not d["v"].any()
    assert np.all((d["g"] >= 0.5) & (d["g"] < 2.0))
    assert not d["g_m"].any() and not d["g_v"].any()
