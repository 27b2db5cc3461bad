"""ctypes declarations of the C ABI in include/sharq.h (one Python name per C entry point)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "lib", "libsharq.so")

NVFP4, MXFP4 = 0, 1
PAIR_4_8, ELEM_2_4, PAIR_4_8_GIVEN, MASK_NONE = 0, 1, 2, 3  # the last two: ablations
F16, BF16, F32 = 0, 1, 2

STATUS = {0: "SHARQ_OK", 1: "SHARQ_ERR_INVALID_ARG", 2: "SHARQ_ERR_UNSUPPORTED",
          3: "SHARQ_ERR_MISALIGNED", 4: "SHARQ_ERR_CUDA", 5: "SHARQ_ERR_TIMEOUT",
          6: "SHARQ_ERR_ARCH"}


class SharqError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"{STATUS.get(code, code)} ({code})")
        self.code = code


class sharq_config(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("mask", ctypes.c_int32), ("residual", ctypes.c_int32)]


class sharq_weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales_dense", ctypes.c_void_p),
                ("scales_sparse", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("cfg", sharq_config)]


class sharq_act(ctypes.Structure):
    _fields_ = [("bq", ctypes.c_void_p), ("bs", ctypes.c_void_p), ("bm", ctypes.c_void_p),
                ("rq", ctypes.c_void_p), ("rs", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("M", ctypes.c_int32), ("K", ctypes.c_int32),
                ("cfg", sharq_config)]


class sharq_act_bytes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("bq", "bs", "bm", "rq", "rs")]


class sharq_weight_bytes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("codes", "scales_dense", "scales_sparse")]


def _load():
    if not os.path.exists(lib_path):
        raise ImportError(
            f"SharQ CUDA library not built ({lib_path} missing); run "
            "`python -m fp4_sparse_dense_b200.build`. There is no CPU fallback.")
    L = ctypes.CDLL(lib_path)
    vp, st = ctypes.c_void_p, ctypes.c_int
    sig = {
        "sharq_act_sizes": (st, [ctypes.c_int32, ctypes.c_int32, sharq_config,
                                 ctypes.POINTER(sharq_act_bytes)]),
        "sharq_weight_sizes": (st, [ctypes.c_int32, ctypes.c_int32, sharq_config,
                                    ctypes.POINTER(sharq_weight_bytes)]),
        "sharq_quantize_weight": (st, [vp, ctypes.c_int, ctypes.POINTER(sharq_weight), vp]),
        "sharq_prepare": (st, [vp, ctypes.c_int, ctypes.POINTER(sharq_act), vp]),
        "sharq_prepare_alongside": (st, [vp, ctypes.c_int, ctypes.POINTER(sharq_act), vp]),
        "sharq_prepare_given_amax": (st, [vp, ctypes.c_int, vp, ctypes.POINTER(sharq_act), vp]),
        "sharq_prepare_rmsnorm": (st, [vp, vp, ctypes.c_float, ctypes.c_int, vp,
                                       ctypes.POINTER(sharq_act), vp]),
        "sharq_linear": (st, [ctypes.POINTER(sharq_act), ctypes.POINTER(sharq_weight), vp,
                              ctypes.c_int, vp, ctypes.c_size_t, vp]),
        "sharq_linear_workspace_size": (st, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             sharq_config, ctypes.POINTER(ctypes.c_size_t)]),
        "sharq_linear_noalloc": (st, [ctypes.POINTER(sharq_act), ctypes.POINTER(sharq_weight),
                                      vp, ctypes.c_int, vp]),
        "sharq_device_status": (st, []),
        "sharq_read_device_status": (st, [vp]),
        "sharq_wait_probe": (st, [vp, ctypes.c_uint32, ctypes.c_uint64, vp]),
        "sharq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


lib = _load()

sharq_act_sizes = lib.sharq_act_sizes
sharq_weight_sizes = lib.sharq_weight_sizes
sharq_quantize_weight = lib.sharq_quantize_weight
sharq_prepare = lib.sharq_prepare
sharq_prepare_alongside = lib.sharq_prepare_alongside
sharq_prepare_given_amax = lib.sharq_prepare_given_amax
sharq_prepare_rmsnorm = lib.sharq_prepare_rmsnorm
sharq_linear = lib.sharq_linear
sharq_linear_workspace_size = lib.sharq_linear_workspace_size
sharq_linear_noalloc = lib.sharq_linear_noalloc
sharq_device_status = lib.sharq_device_status
sharq_read_device_status = lib.sharq_read_device_status
sharq_wait_probe = lib.sharq_wait_probe
sharq_status_string = lib.sharq_status_string


def check(code: int) -> None:
    if code != 0:
        raise SharqError(code)
