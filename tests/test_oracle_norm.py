"""Pins of the RMSNorm oracle (oracle/norm.py) against facts fixed outside it: closed forms,
exact power-of-two scaling, float64 references within the stated rounding bounds, and a
hand-derived sum where the fixed float32 order decides the result."""
import math

import numpy as np
import pytest

from oracle import norm as N
from oracle import sharq as S

F32 = np.float32


def _heavy(M, K, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4, size=(M, K)).astype(F32)
    return N.round16(x, "bf16")


def test_constant_rows_normalise_to_gamma():
    """x = c (a power of two) and eps = 0: sum = K c^2 exactly, rstd = 1/|c| exactly, so
    y = round16(sign(c) * gamma) = sign(c) * gamma for gamma already in bf16."""
    K = 1024
    gamma = N.round16(np.random.default_rng(1).uniform(0.5, 2.0, K).astype(F32), "bf16")
    for c in (1.0, 4.0, 0.125, -2.0):
        x = np.full((2, K), c, F32)
        y, rstd = N.rmsnorm(x, gamma, 0.0, "bf16")
        assert np.all(rstd == F32(1.0 / abs(c)))
        assert np.array_equal(y, np.sign(c) * np.broadcast_to(gamma, y.shape))


def test_power_of_two_scaling_is_exact():
    """With eps = 0, scaling x by 2^k scales the sum by 4^k, the root by 2^k and rstd by
    2^-k, all exactly: y is bit-identical."""
    x = _heavy(8, 512)
    gamma = N.round16(np.random.default_rng(2).normal(1.0, 0.1, 512).astype(F32), "bf16")
    y0, r0 = N.rmsnorm(x, gamma, 0.0, "bf16")
    for k in (-6, -1, 3, 10):
        y, r = N.rmsnorm((x * F32(2.0 ** k)).astype(F32), gamma, 0.0, "bf16")
        assert np.array_equal(y, y0)
        assert np.array_equal(r, (r0 * F32(2.0 ** -k)).astype(F32))


# half an ulp relative to the value: 8 significant bits (bf16), 11 (f16)
@pytest.mark.parametrize("dtype,half_ulp", [("bf16", 2.0 ** -8), ("f16", 2.0 ** -11)])
def test_close_to_float64_rmsnorm(dtype, half_ulp):
    x = _heavy(16, 4096, seed=3)
    gamma = N.round16(np.random.default_rng(4).normal(1.0, 0.2, 4096).astype(F32), dtype)
    eps = 1e-2  # large enough that dropping it breaks the rstd bound below
    y, rstd = N.rmsnorm(x, gamma, eps, dtype)
    x64 = x.astype(np.float64)
    r64 = 1.0 / np.sqrt((x64 * x64).mean(axis=1) + eps)
    assert np.max(np.abs(rstd / r64 - 1.0)) < 4e-6  # a few float32 roundings
    y64 = x64 * r64[:, None] * gamma[None, :].astype(np.float64)
    # one rounding to the 16-bit dtype (half an ulp; fp16 subnormals: half of 2^-24) after
    # float32 work whose error is dominated by rstd's (bounded above)
    tiny = 2.0 ** -25 if dtype == "f16" else 0.0
    assert np.all(np.abs(y - y64) <= (half_ulp + 5e-6) * np.abs(y64) + tiny)


def test_sum_of_squares_within_float32_bound():
    x = _heavy(4, 14336, seed=5)
    ss = N.sum_of_squares(x)
    for row in range(4):
        exact = math.fsum(float(v) * float(v) for v in x[row])
        assert abs(float(ss[row]) - exact) <= 14336 * 2.0 ** -24 * exact


def test_fixed_order_decides_a_hand_derived_sum():
    """K = 256: x_0 = 4096 (square 2^24), every other element 1. Accumulator 0 holds chunk 0
    (elements 0..7): 2^24 + 1 rounds back to 2^24 seven times. Accumulators 1..31 hold 8
    each. The butterfly adds exactly (the ulp at 2^24 is 2 and every partial is even):
    2^24 + 31 * 8 = 16777464. A plain left-to-right sum would give 2^24."""
    x = np.ones((1, 256), F32)
    x[0, 0] = 4096.0
    assert float(N.sum_of_squares(x)[0]) == 16777464.0


def test_prepare_rmsnorm_is_prepare_of_the_normalised_input():
    x = _heavy(6, 512, seed=6)
    gamma = N.round16(np.random.default_rng(7).normal(1.0, 0.3, 512).astype(F32), "bf16")
    p, y, rstd = N.prepare_rmsnorm(x, gamma, 1e-6, "bf16")
    q = S.prepare(y)
    for k, v in S.act_buffers(q).items():
        assert np.array_equal(S.act_buffers(p)[k], v)
