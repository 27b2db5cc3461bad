"""Pins of the oracle's FP4/FP8 codecs against the format definitions (OCP MX spec,
cited by the SharQ page) and against independent implementations written here."""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats as F


def e2m1_from_bits(c):
    """E2M1 decoded from its bit fields (bias 1, 1 mantissa bit), independent of the table."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = Fraction(m, 2) if e == 0 else Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
    return -mag if s else mag


def e4m3_from_bits(c):
    e, m = (c >> 3) & 0xF, c & 7
    if e == 0:
        return Fraction(m, 8) * Fraction(1, 64)
    return Fraction(2) ** (e - 7) * (1 + Fraction(m, 8))


def test_e2m1_table_matches_bit_fields():
    for c in range(16):
        assert F.e2m1_decode(np.array([c]))[0] == float(e2m1_from_bits(c))
    assert sorted(set(abs(F.e2m1_decode(np.arange(16))))) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e4m3_table_matches_bit_fields_and_spec_constants():
    for c in range(127):
        assert F.E4M3_TABLE[c] == float(e4m3_from_bits(c))
    assert F.E4M3_TABLE[0x7E] == 448.0          # max finite (OCP E4M3)
    assert F.E4M3_TABLE[0x08] == 2.0 ** -6      # min normal
    assert F.E4M3_TABLE[0x01] == 2.0 ** -9      # min subnormal
    assert np.all(np.diff(F.E4M3_TABLE) > 0)


def test_roundtrip_all_codes():
    c16 = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(c16)), c16)  # includes -0 -> 0x8
    c127 = np.arange(127, dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode_unsigned(F.e4m3_decode(c127)), c127)


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    (0.2499, 0), (0.2501, 1), (5.0001, 7), (6.0, 7), (7.0, 7), (1e30, 7),
    (-0.1, 8), (-0.0, 8), (0.0, 0), (-5.0, 14), (-7.0, 15),
])
def test_e2m1_ties_to_even_and_saturation(v, code):
    assert F.e2m1_encode(np.array([v], np.float32))[0] == code


def _rne_brute(v, values):
    """Nearest of `values` (exact Fractions) to v; ties to the even index. Independent
    of the oracle's search: compares every candidate."""
    v = Fraction(float(v))
    best = None
    for i, t in enumerate(values):
        d = abs(v - t)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_e2m1_sweep_against_brute_force():
    mags = [e2m1_from_bits(c) for c in range(8)]
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.uniform(-6, 6, 3000), np.arange(-6, 6.01, 0.125)]).astype(np.float32)
    got = F.e2m1_encode(xs)
    for x, g in zip(xs, got):
        want = _rne_brute(min(abs(x), 6.0), mags) | (8 if np.signbit(x) else 0)
        assert g == want, (x, g, want)


def test_e4m3_sweep_against_bit_rounding():
    """Independent E4M3 encoder: round the float32 mantissa to 3 bits (RNE) by integer
    arithmetic, with the subnormal range handled by a fixed-point grid of 2^-9."""
    def enc(x):
        x = float(x)
        if x >= 448:
            return 0x7E
        if x < 2.0 ** -6:  # subnormal grid m * 2^-9, m in 0..8 (m=8 is the min normal)
            q = Fraction(x) / Fraction(1, 512)
            m = int(q)
            rem = q - m
            if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
                m += 1
            return m  # m == 8 encodes 2^-6 = code 0x08
        bits = np.float32(x).view(np.uint32).item()
        e = ((bits >> 23) & 0xFF) - 127
        man = bits & 0x7FFFFF
        keep, rest = man >> 20, man & 0xFFFFF
        if rest > 0x80000 or (rest == 0x80000 and keep & 1):
            keep += 1
        if keep == 8:
            keep, e = 0, e + 1
        c = ((e + 7) << 3) | keep
        return min(c, 0x7E)

    rng = np.random.default_rng(2)
    xs = np.concatenate([
        rng.uniform(0, 500, 4000), 2.0 ** rng.uniform(-12, 9, 4000),
        F.E4M3_TABLE, (F.E4M3_TABLE[1:] + F.E4M3_TABLE[:-1]) / 2,
    ]).astype(np.float32)
    got = F.e4m3_encode_unsigned(xs)
    for x, g in zip(xs, got):
        assert g == enc(x), (x, g, enc(x))


def test_e8m0_decode():
    assert F.e8m0_decode(np.array([127]))[0] == 1.0
    assert F.e8m0_decode(np.array([0]))[0] == 2.0 ** -127
    assert F.e8m0_decode(np.array([254]))[0] == 2.0 ** 127


def test_bf16_round_matches_torch_on_float32_values():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 10 ** rng.uniform(-5, 5, 20000)]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.bf16_round(x.astype(np.float64)), want)


def test_bf16_round_single_rounding_from_float64():
    # 1 + 2^-8 + 2^-40 lies just above the bf16 midpoint 1 + 2^-8: rounds up to 1 + 2^-7.
    # A float32 first step would land exactly on the midpoint and round to even (1.0).
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert F.bf16_round(np.array([v]))[0] == 1.0 + 2.0 ** -7
    for a, b in itertools.product([1.0, -3.5], [2.0 ** -20, 0.0]):
        assert F.bf16_round(np.array([a + b]))[0] == a
