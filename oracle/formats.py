"""FP4 / FP8 number formats used by SharQ, written out from their definitions.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package; it is
the slow, obviously-correct CPU reference that the CUDA kernels are checked against.

Formats (SharQ page, abstract: "generalizes across NVFP4, HiF4, and MXFP4"; the
encodings themselves are those of the OCP Microscaling (MX) specification that the
page's reference list cites, and of NVIDIA's NVFP4):

* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit. Magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no inf/NaN. Code = sign<<3 | magnitude index.
* E4M3 (FP8, "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
  subnormals (m/8)*2^-6; max finite 448; 0x7F is NaN. Used unsigned as NVFP4 block scale.
* E8M0: 8 exponent bits, value 2^(c-127), c in [0, 254]; MXFP4 block scale.

Rounding is round-to-nearest, ties to the even code, with saturation to the largest
finite value ("satfinite"). Every encoder below works by looking the value up between
its two neighbouring representable values, so the result can be checked by eye.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------- E2M1

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit codes (uint8, low nibble) -> float64 values (sign bit 3, -0 for 0x8)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -mag, mag)


def _nearest_even(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the ascending `table` to each `mag` (ties -> even index).

    `mag` must lie within [table[0], table[-1]]. All arithmetic is float64, in which the
    differences between an fp32 value and a table entry are exact.
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(table, mag, side="left")  # first entry >= mag
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    exact = table[hi] == mag
    d_lo = mag - table[lo]
    d_hi = table[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(exact, hi, idx)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """float32/float64 values -> E2M1 codes, RNE, saturating at +-6; sign kept (-0 -> 0x8)."""
    x = np.asarray(x, dtype=np.float64)
    assert not np.any(np.isnan(x)), "E2M1 has no NaN"
    mag = np.minimum(np.abs(x), E2M1_MAX)
    idx = _nearest_even(mag, E2M1_MAGNITUDES).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 3
    return (idx | sign).astype(np.uint8)


# ----------------------------------------------------------------------------- E4M3


def _e4m3_table() -> np.ndarray:
    """Values of the non-negative finite E4M3 codes 0x00..0x7E (ascending with the code)."""
    vals = np.zeros(127, dtype=np.float64)
    for c in range(127):
        e = (c >> 3) & 0xF
        m = c & 7
        if e == 0:
            vals[c] = (m / 8.0) * 2.0 ** (-6)
        else:
            vals[c] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_TABLE = _e4m3_table()
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Unsigned use (scales): code 0x00..0x7E -> float64. Sign bit honoured if set."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    mag = c & 0x7F
    assert not np.any(mag == 0x7F), "E4M3 NaN code"
    v = E4M3_TABLE[mag]
    return np.where(c & 0x80, -v, v)


def e4m3_encode_unsigned(x: np.ndarray) -> np.ndarray:
    """Non-negative float -> E4M3 code (RNE, ties to even code, satfinite at 448; +inf -> 448)."""
    x = np.asarray(x, dtype=np.float64)
    assert not np.any(np.isnan(x)) and np.all(x >= 0)
    mag = np.minimum(x, E4M3_MAX)
    return _nearest_even(mag, E4M3_TABLE).astype(np.uint8)


# ----------------------------------------------------------------------------- E8M0


def e8m0_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64)
    assert np.all((c >= 0) & (c <= 254)), "E8M0 NaN code"
    return np.ldexp(1.0, c - 127)


# ----------------------------------------------------------------------------- bf16


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    Rounds once, directly from the float64 value (no intermediate float32 rounding).
    Assumes values within the normal bf16 range or zero.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    m, e = np.frexp(x[nz])  # x = m * 2^e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits: scale mantissa to [128, 256) and round half-even
    q = np.rint(m * 256.0)  # numpy rint rounds half to even
    out[nz] = np.ldexp(q, e - 8)
    return out
