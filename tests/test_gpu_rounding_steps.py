"""The correctly rounded float32 reciprocal, quotient and square root that
the SwiGLU gate kernels and the optimizer updates compute from the
approximate hardware reciprocal (root) and fused multiply-adds (Markstein's
correction steps), checked through the testing hooks against the IEEE
results numpy computes: the reciprocal and the square root for every float32
significand at several exponents, the quotient on random operands over the
steps' range and on edge cases that take the IEEE fallback."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import int8_quantized_act_b200 as ql
from parity_util import dev, host

pytestmark = pytest.mark.gpu


def _divrn(a, d):
    ta, td = dev(a), dev(d)
    q, y = torch.empty_like(ta), torch.empty_like(ta)
    ql.ql_test_divrn(ta, td, q, y)
    return host(q), host(y)


def _sqrtrn(v):
    tv = dev(v)
    s0, s1 = torch.empty_like(tv), torch.empty_like(tv)
    ql.ql_test_sqrtrn(tv, s0, s1)
    return host(s0), host(s1)


def _bits_equal(x, ref):
    """Bit for bit, every NaN counting as equal to every NaN."""
    xb, rb = x.view(np.uint32), ref.view(np.uint32)
    both_nan = np.isnan(x) & np.isnan(ref)
    return np.array_equal(np.where(both_nan, 0, xb), np.where(both_nan, 0, rb))


def _mismatches(x, ref):
    both_nan = np.isnan(x) & np.isnan(ref)
    return int(np.count_nonzero((x.view(np.uint32) != ref.view(np.uint32)) & ~both_nan))


def _significands(exponent):
    """Every float32 with the given unbiased exponent, in order."""
    sig = np.arange(1 << 23, dtype=np.uint32)
    return ((np.uint32(127 + exponent) << np.uint32(23)) | sig).view(np.float32)


@pytest.mark.parametrize("exponent", [0, 1, 7, 12, 23, -20, 40, -59, 59])
def test_reciprocal_steps_every_significand(exponent):
    """y = 1/d equals the IEEE quotient for every significand of d."""
    d = _significands(exponent)
    q, y = _divrn(np.ones_like(d), d)
    ref = np.float32(1.0) / d
    assert _bits_equal(y, ref) and _bits_equal(q, ref)


def test_quotient_steps_random_operands():
    """q = a/d against the IEEE quotient over the gate's range (d = 1 + e^-a
    in [1, 2^24]) and over the wide range the optimizer's a/d takes."""
    rng = np.random.Generator(np.random.PCG64(11))
    n = 1 << 24
    a = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-90, 101, n))).astype(np.float32)
    a *= np.where(rng.random(n) < 0.5, -1, 1).astype(np.float32)
    d = np.minimum((1.0 + np.exp2(rng.uniform(-30, 24, n))), 2.0 ** 24).astype(np.float32)
    q, _ = _divrn(a, d)
    assert _bits_equal(q, a / d)
    a = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-60, 60, n))).astype(np.float32)
    a *= np.where(rng.random(n) < 0.5, -1, 1).astype(np.float32)
    d = (rng.uniform(1, 2, n) * np.exp2(rng.integers(-60, 60, n))).astype(np.float32)
    q, y = _divrn(a, d)
    assert _bits_equal(q, a / d) and _bits_equal(y, np.float32(1) / d)


def test_quotient_steps_edge_operands():
    """All-ones significands, the range ends and past them, zero, subnormal,
    huge, infinite and NaN operands (the IEEE fallback past the range)."""
    ones = np.float32(np.nextafter(np.float32(2), np.float32(0)))  # 1.111...1 (binary)
    edge_a = np.float32([1, -1, ones, -ones, 3, 1e-40, -1e-40, 2.0 ** -60, 2.0 ** -61,
                         2.0 ** 60, 2.0 ** 61, 3e38, np.inf, -np.inf, np.nan, 7, 7, 7, 7, 7, 7])
    edge_d = np.float32([ones, ones, ones, 1, 3, 1.5, 1.5, 1.5, 1.5, 2.0 ** 24, 2.0 ** 24,
                         1, 1, 1, 1, 2.0 ** -60, 2.0 ** -61, 2.0 ** 60, 2.0 ** 61, 0.0, np.inf])
    q, y = _divrn(edge_a, edge_d)
    with np.errstate(divide="ignore", invalid="ignore"):
        assert _bits_equal(q, edge_a / edge_d) and _bits_equal(y, np.float32(1) / edge_d)
    # a zero quotient: the value is zero (its sign may differ)
    q, _ = _divrn(np.float32([0.0, -0.0]), np.float32([3.0, 3.0]))
    assert np.array_equal(q, np.float32([0.0, 0.0]))


@pytest.mark.parametrize("exponent", [0, -100, -60, -20, 40, 98])
def test_square_root_steps_every_significand(exponent):
    """sqrt(v), plain and refined form, equals the IEEE square root for every
    v with exponent `exponent` or `exponent + 1` (the root's pattern repeats
    every two exponents)."""
    sig = np.arange(1 << 24, dtype=np.uint32)
    v = ((np.uint32(127 + exponent) << np.uint32(23)) + sig).view(np.float32)
    s0, s1 = _sqrtrn(v)
    ref = np.sqrt(v)
    assert _mismatches(s0, ref) == 0 and _mismatches(s1, ref) == 0


def test_square_root_steps_edge_values():
    """Zero of either sign, the range ends and past them (the IEEE
    fallback), subnormal, negative, infinite and NaN values."""
    v = np.float32([0.0, -0.0, 2.0 ** -100, 2.0 ** -101, 2.0 ** 100, 2.0 ** 101, 1e-40,
                    -1.0, np.inf, np.nan, 3e38, 1.0])
    s0, s1 = _sqrtrn(v)
    with np.errstate(invalid="ignore"):
        ref = np.sqrt(v)
    assert _bits_equal(s0, ref) and _bits_equal(s1, ref)
