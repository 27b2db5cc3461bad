"""CPU oracle of the RMSNorm that the SharQ preparation absorbs.

TEST INFRASTRUCTURE ONLY: imported by tests/ and bench.py's reference leg, never by the
product path; it shares no code with the CUDA kernels.

The SharQ page ("SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
Inference", pith.science 2606.26587; arXiv abstract and "Core claim") states that the fused
preparation operator absorbs layer normalisation together with mask generation and
residual construction. The models it evaluates (Llama-3.1-8B, Qwen2.5/Qwen3) normalise the
input of their attention and MLP projections with RMSNorm, so this module takes that
reading:

    rstd = 1 / sqrt(mean_k x_k^2 + eps)          (per row, float32)
    y_k  = round16((x_k * rstd) * gamma_k)       (float32 products, then the input dtype)

and the preparation then runs on y exactly as on any other input. Rounding y to the 16-bit
activation dtype makes the fused path produce the same bytes as normalising first and
preparing the stored result.

The pages fix no arithmetic, so the float32 order is a reading too. Every operation
rounds to nearest even once; the sum of squares uses this fixed order:

* the row is cut into chunks of 8 consecutive elements; chunk c belongs to accumulator
  c mod 32, and each of the 32 accumulators adds its chunks' squares in increasing k;
* the 32 accumulators are then combined by a butterfly: for off = 16, 8, 4, 2, 1 every
  accumulator a becomes a + (the accumulator at index a XOR off).

The square of a 16-bit input is exact in float32, so only the additions round.
mean = sum / K is one division; rstd = 1 / sqrt(mean + eps) is one addition, one correctly
rounded square root and one division.
"""
from __future__ import annotations

import numpy as np

from oracle import sharq as S

F32 = np.float32
LANES = 32
CHUNK = 8


def sum_of_squares(x: np.ndarray) -> np.ndarray:
    """Per-row sum of x^2 in the fixed float32 order above. x: [M, K], K % 256 == 0."""
    x = np.asarray(x, F32)
    M, K = x.shape
    assert K % (LANES * CHUNK) == 0
    sq = (x * x).astype(F32)
    c = sq.reshape(M, K // (LANES * CHUNK), LANES, CHUNK)  # chunk index j * 32 + lane
    acc = np.zeros((M, LANES), F32)
    for j in range(c.shape[1]):
        for e in range(CHUNK):
            acc = (acc + c[:, j, :, e]).astype(F32)
    lane = np.arange(LANES)
    for off in (16, 8, 4, 2, 1):
        acc = (acc + acc[:, lane ^ off]).astype(F32)
    return acc[:, 0]


def rstd_of(x: np.ndarray, eps: float) -> np.ndarray:
    """Per-row 1 / sqrt(mean(x^2) + eps), float32, one rounding per operation."""
    K = np.asarray(x).shape[1]
    ms = (sum_of_squares(x) / F32(K)).astype(F32)
    root = np.sqrt((ms + F32(eps)).astype(F32)).astype(F32)
    return (F32(1.0) / root).astype(F32)


def round16(v: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the activation dtype ("bf16" or "f16"), nearest even."""
    v = np.asarray(v, F32)
    if dtype == "bf16":
        # bf16 is the top half of the float32 pattern: round that pattern at bit 16,
        # nearest with ties to even (subnormals and overflow to inf included)
        b = np.ascontiguousarray(v).view(np.uint32).astype(np.uint64)
        b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
        return b.astype(np.uint32).view(F32)
    if dtype == "f16":
        return v.astype(np.float16).astype(F32)
    raise ValueError(dtype)


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float, dtype: str):
    """Returns (y [M, K] float32 holding dtype values, rstd [M] float32)."""
    x = np.asarray(x, F32)
    rstd = rstd_of(x, eps)
    t = (x * rstd[:, None]).astype(F32)
    y = (t * np.asarray(gamma, F32)[None, :]).astype(F32)
    return round16(y, dtype), rstd


def prepare_rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float, dtype: str,
                    fmt: str = S.NVFP4, mask: str = S.PAIR48, residual: bool = True,
                    amax=None):
    """The preparation of rmsnorm(x): (Prepared, y, rstd)."""
    y, rstd = rmsnorm(x, gamma, eps, dtype)
    return S.prepare(y, fmt, mask, residual=residual, amax=amax), y, rstd
