"""SharQ sparse-dense FP4 linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/sharq.h`` (library ``lib/libsharq.so``,
built in-tree by ``fp4_sparse_dense_b200.build``). Every step of the path runs in the
library's CUDA kernels; this module only marshals arguments and allocates the caller-owned
buffers with torch. There is no CPU fallback: if the library is missing or the device is
not an sm_100 GPU the calls raise.

Low-level names mirror the C entry points (``sharq_prepare``, ``sharq_linear`` ...);
``quantize_weight``, ``prepare`` and ``linear`` are the tensor-level conveniences.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

from ._abi import (  # noqa: F401
    ELEM_2_4, F16, F32, BF16, MASK_NONE, MXFP4, NVFP4, PAIR_4_8, PAIR_4_8_GIVEN, SharqError, lib,
    lib_path,
    sharq_act, sharq_act_bytes, sharq_config, sharq_weight, sharq_weight_bytes, check,
    sharq_act_sizes, sharq_weight_sizes, sharq_status_string, sharq_device_status,
    sharq_read_device_status,
    sharq_prepare, sharq_quantize_weight, sharq_linear, sharq_linear_workspace_size,
    sharq_linear_noalloc, sharq_prepare_rmsnorm, sharq_wait_probe, sharq_prepare_alongside,
    sharq_prepare_given_amax,
)

__all__ = [
    "Config", "QuantWeight", "PreparedAct", "quantize_weight", "prepare", "prepare_rmsnorm",
    "linear", "sharq_prepare_rmsnorm", "sharq_prepare_alongside", "sharq_prepare_given_amax",
    "sharq_act_sizes", "sharq_weight_sizes", "sharq_prepare", "sharq_quantize_weight",
    "sharq_linear", "sharq_linear_workspace_size", "sharq_linear_noalloc", "sharq_device_status",
    "sharq_read_device_status",
    "sharq_status_string", "SharqError", "linear_workspace",
    "NVFP4", "MXFP4", "PAIR_4_8", "ELEM_2_4", "F16", "BF16", "F32",
]


@dataclass(frozen=True)
class Config:
    """fmt, mask and residual mode of sharq_config. residual: True (the method), False,
    "unquantized" (ablation: residual against the unquantised backbone) or "own" (the
    residual with its own tensor scale, two accumulators; NVFP4 with a pair mask). Masks
    "pair48_given" and "none" are ablations (see include/sharq.h)."""
    fmt: int = NVFP4
    mask: int = PAIR_4_8
    residual: bool | str = True

    def c(self) -> sharq_config:
        if self.residual == "unquantized":
            r = 2
        elif self.residual == "own":
            r = 3
        else:
            r = 1 if self.residual else 0
        return sharq_config(self.fmt, self.mask, r)

    @staticmethod
    def from_names(fmt: str = "nvfp4", mask: str = "pair48", residual: bool | str = True) -> "Config":
        return Config({"nvfp4": NVFP4, "mxfp4": MXFP4}[fmt],
                      {"pair48": PAIR_4_8, "elem24": ELEM_2_4, "pair48_given": PAIR_4_8_GIVEN,
                       "none": MASK_NONE}[mask], residual)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"unsupported input dtype {t.dtype} (need bfloat16 or float16)")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream, device=None):
    """The cudaStream_t of `stream`, or of the current stream of `device` (a torch.device)."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    torch = _torch()
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None and device is not None and device.index is not None:
        return ctypes.c_void_p(raw(device.index))  # no Stream object per call
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class _CStructCache:
    """Caches the ctypes struct a buffer set passes to the C ABI; any field assignment
    drops it, so the struct always holds the current buffers' addresses."""

    def __setattr__(self, name, value):
        if name != "_c":
            self.__dict__.pop("_c", None)
        object.__setattr__(self, name, value)

    def c(self):
        cs = self.__dict__.get("_c")
        if cs is None:
            cs = self._make_c()
            self.__dict__["_c"] = cs
        return cs


@dataclass
class QuantWeight(_CStructCache):
    codes: object
    scales_dense: object
    scales_sparse: object
    tensor_scale: object
    K: int
    N: int
    cfg: Config

    def _make_c(self) -> sharq_weight:
        return sharq_weight(_ptr(self.codes), _ptr(self.scales_dense), _ptr(self.scales_sparse),
                            _ptr(self.tensor_scale), self.K, self.N, self.cfg.c())


@dataclass
class PreparedAct(_CStructCache):
    bq: object
    bs: object
    bm: object
    rq: object
    rs: object
    tensor_scale: object
    M: int
    K: int
    cfg: Config

    def _make_c(self) -> sharq_act:
        return sharq_act(_ptr(self.bq), _ptr(self.bs), _ptr(self.bm), _ptr(self.rq), _ptr(self.rs),
                         _ptr(self.tensor_scale), self.M, self.K, self.cfg.c())


def _u8(n: int, device):
    torch = _torch()
    # 16-byte minimum so that every buffer has a valid, aligned address
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


def empty_weight(K: int, N: int, cfg: Config, device="cuda") -> QuantWeight:
    torch = _torch()
    sz = sharq_weight_bytes()
    check(sharq_weight_sizes(K, N, cfg.c(), ctypes.byref(sz)))
    return QuantWeight(_u8(sz.codes, device), _u8(sz.scales_dense, device),
                       _u8(sz.scales_sparse, device) if sz.scales_sparse else None,
                       torch.zeros(4, dtype=torch.float32, device=device), K, N, cfg)


def empty_act(M: int, K: int, cfg: Config, device="cuda") -> PreparedAct:
    torch = _torch()
    sz = sharq_act_bytes()
    check(sharq_act_sizes(M, K, cfg.c(), ctypes.byref(sz)))
    return PreparedAct(_u8(sz.bq, device), _u8(sz.bs, device),
                       _u8(sz.bm, device) if sz.bm else None,
                       _u8(sz.rq, device) if sz.rq else None,
                       _u8(sz.rs, device) if sz.rs else None,
                       torch.zeros(8, dtype=torch.float32, device=device), M, K, cfg)


def quantize_weight(W, cfg: Config = Config(), out: QuantWeight | None = None,
                    stream=None) -> QuantWeight:
    """W: CUDA tensor [K x N] (bf16/fp16) -> FP4 weight payload with both scale views."""
    K, N = W.shape
    W = W.contiguous()
    out = out or empty_weight(K, N, cfg, W.device)
    cw = out.c()
    check(sharq_quantize_weight(_ptr(W), _dtype_code(W), ctypes.byref(cw), _stream(stream)))
    return out


def prepare(X, cfg: Config = Config(), out: PreparedAct | None = None, stream=None,
            alongside: bool = False, amax=None) -> PreparedAct:
    """X: CUDA tensor [M x K] (bf16/fp16) -> backbone / residual FP4 operands.
    alongside=True: launched to share the GPU with a GEMM running on another stream
    (sharq_prepare_alongside; identical results). amax: a float32 CUDA tensor of one element,
    the NVFP4 tensor amax to use instead of max |X| (sharq_prepare_given_amax)."""
    M, K = X.shape
    if not X.is_contiguous():
        X = X.contiguous()
    out = out or empty_act(M, K, cfg, X.device)
    ca = out.c()
    if amax is not None:
        check(sharq_prepare_given_amax(_ptr(X), _dtype_code(X), _ptr(amax), ctypes.byref(ca),
                                       _stream(stream, X.device)))
        return out
    fn = sharq_prepare_alongside if alongside else sharq_prepare
    check(fn(_ptr(X), _dtype_code(X), ctypes.byref(ca), _stream(stream, X.device)))
    return out


def prepare_rmsnorm(X, gamma, eps: float, cfg: Config = Config(), out: PreparedAct | None = None,
                    rstd=None, stream=None):
    """Prepare RMSNorm(X) with weight gamma [K] (same dtype as X): returns (act, rstd [M])."""
    torch = _torch()
    M, K = X.shape
    X = X.contiguous()
    gamma = gamma.contiguous()
    if gamma.dtype != X.dtype or gamma.numel() != K:
        raise ValueError("gamma must be [K] in the dtype of X")
    out = out or empty_act(M, K, cfg, X.device)
    if rstd is None:
        rstd = torch.empty(M, dtype=torch.float32, device=X.device)
    ca = out.c()
    check(sharq_prepare_rmsnorm(_ptr(X), _ptr(gamma), float(eps), _dtype_code(X), _ptr(rstd),
                                ctypes.byref(ca), _stream(stream)))
    return out, rstd


_WS_BYTES = {}  # (M, N, K, cfg, device) -> bytes the shape's split-K wants


def linear_workspace(M: int, N: int, K: int, cfg: Config = Config(), device="cuda"):
    """Caller-owned split-K workspace for sharq_linear (None when the shape does not split)."""
    key = (M, N, K, cfg, str(device))
    n = _WS_BYTES.get(key)
    if n is None:
        nbytes = ctypes.c_size_t(0)
        check(sharq_linear_workspace_size(M, N, K, cfg.c(), ctypes.byref(nbytes)))
        n = _WS_BYTES[key] = nbytes.value
    return _u8(n, device) if n else None


def linear(act: PreparedAct, w: QuantWeight, out=None, out_dtype=None, workspace="auto",
           stream=None):
    """Y[M x N] = sparse-FP4-GEMM(backbone, W) + dense-FP4-GEMM(residual, W).

    workspace: "auto" allocates the split-K workspace this shape wants (a torch buffer the
    caller may keep and pass again), None runs without splitting K, or a uint8 CUDA tensor.
    """
    torch = _torch()
    if out is None:
        out = torch.empty(act.M, w.N, dtype=out_dtype or torch.bfloat16, device=act.bq.device)
    if out.dtype == torch.bfloat16:
        code = BF16
    elif out.dtype == torch.float32:
        code = F32
    else:
        raise TypeError(f"unsupported output dtype {out.dtype} (need bfloat16 or float32)")
    if isinstance(workspace, str):
        workspace = linear_workspace(act.M, w.N, act.K, act.cfg, act.bq.device)
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() if workspace is not None else 0
    ca, cw = act.c(), w.c()
    check(sharq_linear(ctypes.byref(ca), ctypes.byref(cw), _ptr(out), code, ws_ptr, ws_bytes,
                       _stream(stream, out.device)))
    return out
