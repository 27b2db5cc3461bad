"""Seeded synthetic inputs for the SharQ linear layer (activations X and weights W).

This module is shared by the CPU oracle, the tests and the benchmark. It holds no
arithmetic of the method itself (no masking, no quantisation, no GEMM): it only draws
random numbers and rounds them to the 16-bit input dtype, so that both sides of every
parity check consume identical inputs.

The shapes and value distributions follow the workloads the SharQ page describes
("SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference",
pith.science 2606.26587, abstract and Fig. 3/4 captions): LLM linear layers whose
activations carry a few input-dependent outlier channels on top of a heavy-tailed
bulk. The pages evaluate on Llama-3.1-8B / Qwen models with real data; neither trained
weights nor datasets are used here, so these generators stand in for them:

* ``tiny``: X[16x256] ~ N(0,1) with 4 fixed channels scaled by 30, W ~ N(0, 0.02), fp16.
* ``heavy``: X rows are Student-t(nu=4); 0.5 % of the channels (fixed per tensor)
  are multiplied by a per-channel factor drawn from U[20, 50]; bf16.
* ``heavy_per_row``: like ``heavy`` but the outlier channel set is redrawn per row.
* W ~ N(0, 0.02) for every linear.

Every array is returned as float32 holding values that are exactly representable in
the requested 16-bit dtype (the bf16/fp16 rounding is round-to-nearest-even), together
with the raw 16-bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BF16 = "bf16"
F16 = "f16"


def round_to_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bfloat16 (nearest, ties to even).

    Returns (values as float32, raw uint16 bit patterns). Inputs must be finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert np.all(np.isfinite(x))
    # uint32 arithmetic cannot overflow: finite patterns are <= 0xFF7FFFFF
    b = x.view(np.uint32)
    t = (b >> 16) & 1
    t += 0x7FFF
    t += b
    t >>= 16
    r = t.astype(np.uint16)
    t <<= 16
    return t.view(np.float32), r


def round_to_f16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to IEEE half (numpy's conversion is round-to-nearest-even)."""
    h = np.ascontiguousarray(x, dtype=np.float32).astype(np.float16)
    assert np.all(np.isfinite(h))
    return h.astype(np.float32), h.view(np.uint16)


def to_dtype(x: np.ndarray, dtype: str) -> tuple[np.ndarray, np.ndarray]:
    if dtype == BF16:
        return round_to_bf16(x)
    if dtype == F16:
        return round_to_f16(x)
    raise ValueError(dtype)


@dataclass
class Tensor16:
    """A 16-bit tensor: float32 view of its values plus the raw bit pattern."""

    values: np.ndarray  # float32, exactly representable in `dtype`
    bits: np.ndarray  # uint16
    dtype: str

    @property
    def shape(self):
        return self.values.shape


def to_device(t16: Tensor16, device="cuda"):
    """A Tensor16 as a torch tensor of its 16-bit dtype on `device`, bit-identical (the raw
    patterns are reinterpreted, never converted). torch is imported only here."""
    import torch
    dt = torch.bfloat16 if t16.dtype == BF16 else torch.float16
    bits = np.ascontiguousarray(t16.bits).view(np.int16).copy()
    return torch.from_numpy(bits).view(dt).to(device)


def _mk(x: np.ndarray, dtype: str) -> Tensor16:
    v, b = to_dtype(x, dtype)
    return Tensor16(v, b, dtype)


def gaussian_weight(rng: np.random.Generator, K: int, N: int, dtype: str = BF16,
                    sigma: float = 0.02) -> Tensor16:
    """W[K x N] ~ N(0, sigma^2): the layer's weight, input features along rows."""
    w = rng.standard_normal((K, N), dtype=np.float32)
    w *= np.float32(sigma)
    return _mk(w, dtype)


def tiny_activations(M: int = 16, K: int = 256, seed: int = 0, n_outliers: int = 4,
                     gain: float = 30.0, dtype: str = F16) -> Tensor16:
    """X ~ N(0,1) with `n_outliers` channels (chosen once from a seed-0 stream) x gain."""
    chans = np.random.default_rng(0).choice(K, n_outliers, replace=False)
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(M, K)).astype(np.float32)
    x[:, chans] *= np.float32(gain)
    return _mk(x, dtype)


def heavy_activations(rng: np.random.Generator, M: int, K: int, *, per_row: bool = False,
                      frac: float = 0.005, lo: float = 20.0, hi: float = 50.0,
                      nu: float = 4.0, dtype: str = BF16) -> Tensor16:
    """Student-t(nu) rows with a fraction `frac` of outlier channels scaled by U[lo, hi].

    With per_row=False the outlier channel set (and its gains) is fixed for the whole
    tensor; with per_row=True every row draws its own channel set and gains.
    """
    x = rng.standard_t(nu, size=(M, K)).astype(np.float32)
    n_out = max(1, int(round(frac * K)))
    if not per_row:
        chans = rng.choice(K, n_out, replace=False)
        gains = rng.uniform(lo, hi, size=n_out).astype(np.float32)
        x[:, chans] *= gains[None, :]
    else:
        for m in range(M):
            chans = rng.choice(K, n_out, replace=False)
            x[m, chans] *= rng.uniform(lo, hi, size=n_out).astype(np.float32)
    return _mk(x, dtype)


# ----------------------------------------------------------------------------------
# Named workloads (the five configurations of the benchmark plan)
# ----------------------------------------------------------------------------------

LLAMA8B_LINEARS = (  # name, K (in), N (out)
    ("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024), ("o", 4096, 4096),
    ("gate", 4096, 14336), ("up", 4096, 14336), ("down", 14336, 4096),
)


@dataclass
class Problem:
    name: str
    M: int
    K: int
    N: int
    fmt: str  # "nvfp4" | "mxfp4"
    mask: str  # "pair48" | "elem24"
    dtype: str
    seed: int
    per_row: bool = False
    kind: str = "heavy"  # "heavy" | "tiny"
    extra: dict = field(default_factory=dict)

    def make(self) -> tuple[Tensor16, Tensor16]:
        """Draw (X[M x K], W[K x N]) for this problem."""
        if self.kind == "tiny":
            x = tiny_activations(self.M, self.K, seed=self.seed, dtype=self.dtype)
            w = gaussian_weight(np.random.default_rng(self.seed + 1), self.K, self.N, self.dtype)
            return x, w
        rng = np.random.default_rng(self.seed)
        x = heavy_activations(rng, self.M, self.K, per_row=self.per_row, dtype=self.dtype)
        if "w_seed" in self.extra:  # layer stack: each linear's weight has its own stream
            rng = np.random.default_rng(100_000 + self.extra["w_seed"])
        w = gaussian_weight(rng, self.K, self.N, self.dtype)
        return x, w

    def make_x(self) -> Tensor16:
        return self.make()[0] if self.kind == "tiny" else heavy_activations(
            np.random.default_rng(self.seed), self.M, self.K, per_row=self.per_row, dtype=self.dtype)


def config_problems(index: int, M: int | None = None, fmt: str = "nvfp4") -> list[Problem]:
    """Problems of benchmark configuration `index` (1..5); seeds = index*1000 + M."""
    if index == 1:
        return [Problem("tiny_16x256x128", 16, 256, 128, "nvfp4", "elem24", F16, 0, kind="tiny")]
    if index == 2:
        return [Problem("attn_proj_2048x4096x4096", 2048, 4096, 4096, "nvfp4", "pair48", BF16, 2000 + 2048)]
    if index == 3:
        return [Problem("mlp_gate_up_4096x4096x14336", 4096, 4096, 14336, "nvfp4", "pair48", BF16,
                        3000 + 4096)]
    if index == 4:
        Ms = [1, 8, 16, 64, 4096] if M is None else [M]
        return [Problem(f"mlp_down_{m}x14336x4096", m, 14336, 4096, "nvfp4", "pair48", BF16,
                        4000 + m, per_row=True) for m in Ms]
    if index == 5:
        Ms = [1 << i for i in range(14)] if M is None else [M]
        out = []
        for m in Ms:
            for layer in range(32):
                for idx, (nm, k, n) in enumerate(LLAMA8B_LINEARS):
                    out.append(Problem(f"l{layer}.{nm}_{m}x{k}x{n}", m, k, n, fmt, "pair48", BF16,
                                       5000 + m, extra={"layer": layer, "idx": idx,
                                                        "w_seed": layer * 7 + idx}))
        return out
    raise ValueError(index)
