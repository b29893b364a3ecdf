"""Seeded synthetic inputs for the INT8 quantized-training Linear layer.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantization, rotation, GEMM or update).  Both the CPU
oracle (``oracle/``) and the CUDA path (``int8_quantized_act_b200``) receive
the arrays it returns, so the two sides always see identical bytes.

Shapes and distributions follow the five workloads used for parity and
measurement:

* ``tiny``      M=32, K=256, N=128, fp32, Hadamard block 256, channels 0..3 x20.
* ``rotated``   the 5376 -> 7168 layer of the OneTrainer PR "Int8 conv rot"
                (#1681, commit note item 1 timing table), bf16 X with 1% of
                the input channels scaled x30, Hadamard block 128.
* ``swiglu``    d_model 4096, d_ff 14336, 8192 tokens.
* ``update``    int8 weight matrices [n, n] for the stochastic-requant update.

All floating draws are float32 from numpy's PCG64 generator.  bf16 inputs are
produced by rounding the float32 draw to bf16 (round-to-nearest-even, done by
torch's CPU cast); the oracle receives the exact float32 upcast of those bf16
values, so both sides quantize the same numbers.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "normal",
    "uniform",
    "outlier_channels",
    "to_bf16",
    "tiny_layer",
    "rotated_layer",
    "swiglu_mlp",
    "swiglu_stage_inputs",
    "update_state",
]


def normal(shape, std: float, seed: int) -> np.ndarray:
    """float32 array ~ N(0, std^2), drawn from PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def uniform(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    """float32 array ~ U(lo, hi), drawn from PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.uniform(lo, hi, size=shape).astype(np.float32)


def outlier_channels(n_cols: int, fraction: float, seed: int) -> np.ndarray:
    """Sorted indices of round(fraction * n_cols) input channels, chosen by a
    seeded permutation (the outlier channels that a rotation spreads out)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    count = int(round(fraction * n_cols))
    return np.sort(rng.permutation(n_cols)[:count])


def to_bf16(x: np.ndarray):
    """Round a float32 array to bf16.

    Returns ``(t, x32)`` where ``t`` is a CPU ``torch.bfloat16`` tensor and
    ``x32`` is its exact float32 upcast as a numpy array.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)
    return t, t.float().numpy()


def tiny_layer(seed: int = 0) -> dict:
    """The small single-layer case: X fp32 [32,256] ~N(0,1) with channels 0..3
    scaled x20, W fp32 [128,256] ~N(0,0.02), bias ~N(0,0.01), dY ~N(0,1)
    [32,128]; Hadamard block 256; one SGD (lr 1e-2) stochastic-round step."""
    M, K, N = 32, 256, 128
    x = normal((M, K), 1.0, seed + 1)
    x[:, 0:4] *= np.float32(20.0)
    return {
        "M": M, "K": K, "N": N, "block": 256,
        "x": x,
        "w": normal((N, K), 0.02, seed + 2),
        "bias": normal((N,), 0.01, seed + 3),
        "dy": normal((M, N), 1.0, seed + 4),
        "lr": 1e-2, "seed": seed, "step": 1,
    }


def rotated_layer(M: int = 2048, seed: int = 0, with_dy: bool = True,
                  K: int = 5376, N: int = 7168) -> dict:
    """The 5376 -> 7168 layer: X ~N(0,1) [M,K] with 1% of the K channels
    (chosen by a seed-0 permutation) scaled x30, rounded to bf16; W ~N(0,0.02)
    [N,K] fp32; bias ~N(0,0.01); dY ~N(0,1) [M,N] rounded to bf16.
    Hadamard block 128 (5376 = 42 x 128)."""
    x = normal((M, K), 1.0, seed + 11)
    ch = outlier_channels(K, 0.01, 0)
    x[:, ch] *= np.float32(30.0)
    x_bf, x32 = to_bf16(x)
    out = {
        "M": M, "K": K, "N": N, "block": 128,
        "x_bf16": x_bf, "x": x32, "outliers": ch,
        "w": normal((N, K), 0.02, seed + 12),
        "bias": normal((N,), 0.01, seed + 13),
    }
    if with_dy:
        dy_bf, dy32 = to_bf16(normal((M, N), 1.0, seed + 14))
        out["dy_bf16"], out["dy"] = dy_bf, dy32
    return out


def swiglu_mlp(T: int = 8192, d_model: int = 4096, d_ff: int = 14336,
               seed: int = 0) -> dict:
    """SwiGLU MLP step: X ~N(0,1) [T,d_model] bf16; w1, w3 [d_ff,d_model] and
    w2 [d_model,d_ff] ~N(0,0.02); dY ~N(0,1) [T,d_model] bf16; AdamW lr 1e-3."""
    x_bf, x32 = to_bf16(normal((T, d_model), 1.0, seed + 21))
    dy_bf, dy32 = to_bf16(normal((T, d_model), 1.0, seed + 25))
    return {
        "T": T, "d_model": d_model, "d_ff": d_ff,
        "x_bf16": x_bf, "x": x32,
        "w1": normal((d_ff, d_model), 0.02, seed + 22),
        "w3": normal((d_ff, d_model), 0.02, seed + 23),
        "w2": normal((d_model, d_ff), 0.02, seed + 24),
        "dy_bf16": dy_bf, "dy": dy32,
        "lr": 1e-3,
    }


def swiglu_gate_inputs(T: int = 8192, d_ff: int = 14336, seed: int = 0) -> dict:
    """Inputs of the SwiGLU gate and of the calls around it, drawn directly
    (so that each step can be checked on its own): the stacked
    pre-activations ab = [a | b] [T, 2 d_ff] ~N(0, 1.28^2) (the spread of
    X W^T for X ~N(0,1), W ~N(0,0.02), d_model 4096) and the gradient at h,
    dh [T, d_ff] ~N(0, 1.28^2), each rounded to bf16 (the float32 arrays are
    the exact upcasts)."""
    sd = 0.02 * 64.0
    ab = np.empty((T, 2 * d_ff), np.float32)
    ab[:, :d_ff] = normal((T, d_ff), sd, seed + 41)
    ab[:, d_ff:] = normal((T, d_ff), sd, seed + 42)
    ab_bf, ab32 = to_bf16(ab)
    del ab
    dh_bf, dh32 = to_bf16(normal((T, d_ff), sd, seed + 43))
    return {"ab_bf16": ab_bf, "ab": ab32, "dh_bf16": dh_bf, "dh": dh32}


def update_state(N: int, K: int, seed: int = 0, warm: bool = False,
                 weight_norm: bool = False) -> dict:
    """Inputs of one stochastic-requant update of an int8 [N,K] weight:
    the float weight W ~N(0,0.02) to be prepared, the gradient ~N(0,1e-3),
    AdamW moments (zero at step 1; for a warm start at step 10,
    m ~N(0,1e-4) and v = (N(0,1e-3))^2), and for the row-wise weight-norm
    variant the per-row magnitude g ~U(0.5,2) with zero moments."""
    out = {
        "N": N, "K": K,
        "w": normal((N, K), 0.02, seed + 31),
        "grad": normal((N, K), 1e-3, seed + 32),
        "step": 10 if warm else 1,
    }
    if warm:
        out["m"] = normal((N, K), 1e-4, seed + 33)
        out["v"] = np.square(normal((N, K), 1e-3, seed + 34))
    else:
        out["m"] = np.zeros((N, K), np.float32)
        out["v"] = np.zeros((N, K), np.float32)
    if weight_norm:
        out["g"] = uniform((N,), 0.5, 2.0, seed + 35)
        out["g_m"] = np.zeros((N,), np.float32)
        out["g_v"] = np.zeros((N,), np.float32)
    return out
