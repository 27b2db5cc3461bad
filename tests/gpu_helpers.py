"""Shared code of the GPU parity tests: run the CUDA path through the binding and fetch
its byte buffers; build the oracle's expected bytes for the same seeded inputs."""
from __future__ import annotations

import numpy as np

from oracle import layouts as L
from oracle import sharq as S
from workloads import to_device  # noqa: F401  (re-exported for the tests)

def torch_mod():
    import torch
    return torch


def cfg_of(fmt: str, mask: str, residual: bool = True):
    import fp4_sparse_dense_b200 as sq
    return sq.Config.from_names(fmt, mask, residual)


def act_bytes(act) -> dict:
    out = {"tensor_scale": act.tensor_scale[:1].cpu().numpy(),
           "bq": act.bq.cpu().numpy(), "bs": act.bs.cpu().numpy()}
    if act.bm is not None:
        out["bm"] = act.bm.cpu().numpy()
    if act.rq is not None:
        out["rq"] = act.rq.cpu().numpy()
        out["rs"] = act.rs.cpu().numpy()
    return out


def weight_bytes(w) -> dict:
    out = {"tensor_scale": w.tensor_scale[:1].cpu().numpy(), "codes": w.codes.cpu().numpy(),
           "scales_dense": w.scales_dense.cpu().numpy()}
    if w.scales_sparse is not None:
        out["scales_sparse"] = w.scales_sparse.cpu().numpy()
    return out


def first_mismatch(a: np.ndarray, b: np.ndarray) -> str:
    a = np.asarray(a).reshape(-1)
    b = np.asarray(b).reshape(-1)
    if a.size != b.size:
        return f"size {a.size} != {b.size}"
    bad = np.nonzero(a.view(np.uint8) != b.view(np.uint8))[0] if a.dtype == b.dtype else []
    if len(bad) == 0:
        return "equal"
    i = bad[0]
    return f"{len(bad)} bytes differ; first at byte {i}: got {a.view(np.uint8)[i]:#x} want {b.view(np.uint8)[i]:#x}"


def assert_bytes_equal(got: dict, want: dict, keys=None, n_valid: dict | None = None):
    for k in keys or want:
        g, w = np.asarray(got[k]), np.asarray(want[k])
        if n_valid and k in n_valid:
            g = g.reshape(-1)[:n_valid[k]]
        g = g.reshape(-1)[: w.reshape(-1).size] if g.size >= w.size else g
        assert g.view(np.uint8).tobytes() == w.view(np.uint8).tobytes(), f"{k}: {first_mismatch(g, w)}"


def upload_act(buf: dict, M: int, K: int, cfg, device="cuda"):
    """Oracle act bytes -> a PreparedAct on the GPU (to test the GEMM on its own)."""
    torch = torch_mod()
    import fp4_sparse_dense_b200 as sq
    act = sq.empty_act(M, K, cfg, device)
    for k in ("bq", "bs", "bm", "rq", "rs"):
        if k in buf and getattr(act, k) is not None:
            t = torch.from_numpy(np.ascontiguousarray(buf[k])).to(device)
            getattr(act, k)[: t.numel()].copy_(t)
    act.tensor_scale[:1].copy_(torch.from_numpy(buf["tensor_scale"]).to(device))
    return act


def upload_weight(buf: dict, K: int, N: int, cfg, device="cuda"):
    torch = torch_mod()
    import fp4_sparse_dense_b200 as sq
    w = sq.empty_weight(K, N, cfg, device)
    for k in ("codes", "scales_dense", "scales_sparse"):
        if k in buf and getattr(w, k) is not None:
            t = torch.from_numpy(np.ascontiguousarray(buf[k])).to(device)
            getattr(w, k)[: t.numel()].copy_(t)
    w.tensor_scale[:1].copy_(torch.from_numpy(buf["tensor_scale"]).to(device))
    return w


def rel_fro(got: np.ndarray, want: np.ndarray) -> float:
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(np.asarray(got, np.float64) - want) / (den if den > 0 else 1.0))


def sampled_act_rows(buf: dict, rows: np.ndarray, M: int, K: int, fmt: str, mask: str) -> dict:
    """Extract the canonical per-row values of sampled rows from full-size act bytes."""
    Bb, Br = S.backbone_block(fmt, mask), S.residual_block(fmt)
    bq_w = K // 4 if mask == S.PAIR48 else K // 2
    out = {"bq": buf["bq"].reshape(-1)[: M * bq_w].reshape(M, bq_w)[rows]}
    out["bs"] = L.from_scale_layout(buf["bs"], M, K // Bb)[rows]
    if mask == S.PAIR48:
        out["meta"] = L.from_meta48_layout(buf["bm"], M, K)[rows]
    else:
        out["meta"] = L.unpack_nibbles(buf["bm"].reshape(-1)[: M * K // 8].reshape(M, K // 8))[rows]
    if "rq" in buf:
        out["rq"] = buf["rq"].reshape(-1)[: M * K // 2].reshape(M, K // 2)[rows]
        out["rs"] = L.from_scale_layout(buf["rs"], M, K // Br)[rows]
    return out
