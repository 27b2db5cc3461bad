"""Cost of the weight's 32-element NVFP4 blocks against 16-element ones (oracle only).

TEST INFRASTRUCTURE: a study on the CPU oracle, not part of the product path.

With the pair-wise 4:8 mask the weight is quantised in 32-element blocks so that one FP4
payload is exact under both scale views the two GEMMs read: the sparse block-scaled MMA
applies one scale per 32 logical K, the dense one per 16 ("one FP4 weight payload ...
path-specific scale views": SharQ page, pith.science 2606.26587, abstract). This measures
what that costs against the usual 16-element NVFP4 weight on the same weight and the same
prepared activations:

* the weight's reconstruction error ||W - deq(W)||_F / ||W||_F, and
* the relative Frobenius error of Y against the unquantised product X W (float64), on a
  sample of token rows (rows are independent, so sampling is exact per row).

Usage: python -m oracle.weight_block_study [--rows 64] [--K 4096] [--N 14336]
(the default shape is the MLP gate/up weight W[4096 x 14336] ~ N(0, 0.02)).
"""
from __future__ import annotations

import argparse

import numpy as np

from . import sharq as S


def weight_error(w: np.ndarray, qw: S.QWeight) -> float:
    """||W - deq(W)||_F / ||W||_F, W given [K x N]."""
    deq = S.weight_values(qw).T * float(qw.s_gw)  # [K x N]
    w64 = np.asarray(w, np.float64)
    return float(np.linalg.norm(w64 - deq) / np.linalg.norm(w64))


def study(x: np.ndarray, w: np.ndarray, fmt: str = S.NVFP4, amax_x=None) -> dict:
    """Errors of the method's Y with 32- and 16-element weight blocks. x: [rows x K] (a
    sample of the tensor's rows; amax_x is the whole tensor's max |x|), w: [K x N]."""
    q32 = S.quantize_weight(w, fmt, S.PAIR48)   # the method's weight (32-element blocks)
    q16 = S.quantize_weight(w, fmt, S.ELEM24)   # the same recipe in 16-element blocks
    assert S.weight_block(fmt, S.PAIR48) == 32 and S.weight_block(fmt, S.ELEM24) == 16
    p = S.prepare(x, fmt, S.PAIR48, amax=amax_x)
    y_ref = np.asarray(x, np.float64) @ np.asarray(w, np.float64)
    out = {}
    for name, q in (("32", q32), ("16", q16)):
        y = S.linear(p, q)
        out[name] = {"w_err": weight_error(w, q),
                     "y_err": float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref))}
    # the activation side alone: the method's activations times the unquantised weight
    a = S.backbone_values(p) * float(p.s_g) + p.r_deq.astype(np.float64)
    y_act = a @ np.asarray(w, np.float64)
    out["act_only_y_err"] = float(np.linalg.norm(y_act - y_ref) / np.linalg.norm(y_ref))
    return out


def main():
    from workloads import gaussian_weight, heavy_activations
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=64)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=14336)
    ap.add_argument("--seed", type=int, default=3000 + 4096)
    a = ap.parse_args()
    rng = np.random.default_rng(a.seed)
    x = heavy_activations(rng, 4096, a.K)  # the MLP gate/up activations (fixed outliers)
    w = gaussian_weight(rng, a.K, a.N)
    rows = np.linspace(0, x.values.shape[0] - 1, a.rows).astype(np.int64)
    for fmt in (S.NVFP4,):
        r = study(x.values[rows], w.values, fmt, amax_x=S.amax_of(x.values))
        print(f"{fmt} W[{a.K}x{a.N}], {a.rows} rows: "
              f"weight error 32-block {r['32']['w_err']:.4%}, 16-block {r['16']['w_err']:.4%}; "
              f"Y error 32-block {r['32']['y_err']:.4%}, 16-block {r['16']['y_err']:.4%}; "
              f"activations alone {r['act_only_y_err']:.4%}")


if __name__ == "__main__":
    main()
