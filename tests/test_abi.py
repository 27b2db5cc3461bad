"""CPU checks of the C ABI: the library builds, loads, exports every entry point that
include/sharq.h declares, answers size queries like the oracle's layouts, and rejects bad
arguments with an error code (no GPU is touched)."""
import ctypes
import importlib.util
import os
import re

import numpy as np
import pytest

from oracle import sharq as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    spec = importlib.util.spec_from_file_location(
        "sharq_build", os.path.join(ROOT, "fp4_sparse_dense_b200", "build.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


@pytest.fixture(scope="module")
def sq():
    _build_module().build()
    import fp4_sparse_dense_b200 as sq
    return sq


def _declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "sharq.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(sharq_[a-z_]+)\s*\(", hdr)))


def test_header_declares_entry_points():
    syms = _declared_symbols()
    for name in ("sharq_quantize_weight", "sharq_prepare", "sharq_linear", "sharq_act_sizes",
                 "sharq_weight_sizes", "sharq_device_status", "sharq_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol(sq):
    L = ctypes.CDLL(sq.lib_path)
    for name in _declared_symbols():
        assert hasattr(L, name), name


def test_status_strings(sq):
    assert sq.sharq_status_string(0) == b"SHARQ_OK"
    assert sq.sharq_status_string(5) == b"SHARQ_ERR_TIMEOUT"
    assert sq.sharq_status_string(99) == b"SHARQ_ERR_UNKNOWN"


CFGS = [(f, m, r) for f in ("nvfp4", "mxfp4") for m in ("pair48", "elem24", "pair48_given", "none")
        for r in (True, False)]


@pytest.mark.parametrize("fmt,mask,res", CFGS)
@pytest.mark.parametrize("M,K", [(1, 256), (16, 256), (130, 512), (300, 4096)])
def test_act_sizes_match_oracle_layouts(sq, fmt, mask, res, M, K):
    x = np.random.default_rng(0).standard_normal((M, K)).astype(np.float32)
    given = S.keep_pairs48(x) if mask == "pair48_given" else None
    want = S.act_buffers(S.prepare(x, fmt, mask, residual=res, given=given))
    sz = sq.sharq_act_bytes()
    cfg = sq.Config.from_names(fmt, mask, res).c()
    assert sq.sharq_act_sizes(M, K, cfg, ctypes.byref(sz)) == 0
    assert sz.bq == want["bq"].size and sz.bs == want["bs"].size
    assert sz.bm == (want["bm"].size if "bm" in want else 0)
    if res:
        assert sz.rq == want["rq"].size and sz.rs == want["rs"].size
    else:
        assert sz.rq == 0 and sz.rs == 0


@pytest.mark.parametrize("fmt,mask", [(f, m) for f in ("nvfp4", "mxfp4")
                                      for m in ("pair48", "elem24", "pair48_given", "none")])
def test_weight_sizes_match_oracle_layouts(sq, fmt, mask):
    K, N = 512, 384
    w = np.random.default_rng(1).standard_normal((K, N)).astype(np.float32)
    want = S.weight_buffers(S.quantize_weight(w, fmt, mask))
    sz = sq.sharq_weight_bytes()
    assert sq.sharq_weight_sizes(K, N, sq.Config.from_names(fmt, mask).c(), ctypes.byref(sz)) == 0
    assert sz.codes == want["codes"].size and sz.scales_dense == want["scales_dense"].size
    assert sz.scales_sparse == (want["scales_sparse"].size if S.is_pair(mask) else 0)


@pytest.mark.parametrize("mask", ["pair48", "pair48_given"])
def test_own_residual_scale_sizes_match_oracle_layouts(sq, mask):
    """residual == 3 writes the buffers of residual on (its scale goes to tensor_scale[6])."""
    M, K = 130, 512
    x = np.random.default_rng(2).standard_normal((M, K)).astype(np.float32)
    given = S.keep_pairs48(x) if mask == "pair48_given" else None
    want = S.act_buffers(S.prepare(x, "nvfp4", mask, given=given, residual_scale="own"))
    sz = sq.sharq_act_bytes()
    assert sq.sharq_act_sizes(M, K, sq.Config.from_names("nvfp4", mask, "own").c(),
                              ctypes.byref(sz)) == 0
    assert (sz.bq, sz.bs, sz.bm, sz.rq, sz.rs) == tuple(
        want[k].size for k in ("bq", "bs", "bm", "rq", "rs"))


def test_bad_shapes_and_configs_rejected(sq):
    sz = sq.sharq_act_bytes()
    ok = sq.Config().c()
    assert sq.sharq_act_sizes(16, 200, ok, ctypes.byref(sz)) == 1   # K % 256
    assert sq.sharq_act_sizes(0, 256, ok, ctypes.byref(sz)) == 1    # M < 1
    assert sq.sharq_act_sizes(16, 256, sq.sharq_config(7, 0, 1), ctypes.byref(sz)) == 1
    assert sq.sharq_act_sizes(16, 256, sq.sharq_config(0, 0, 4), ctypes.byref(sz)) == 1
    assert sq.sharq_act_sizes(16, 256, sq.sharq_config(0, 4, 1), ctypes.byref(sz)) == 1
    # the residual's own tensor scale: NVFP4 with a pair mask only
    for fmt, mask, code in ((0, 0, 0), (0, 2, 0), (1, 0, 2), (0, 1, 2), (0, 3, 2)):
        assert sq.sharq_act_sizes(16, 256, sq.sharq_config(fmt, mask, 3), ctypes.byref(sz)) == code
    wz = sq.sharq_weight_bytes()
    assert sq.sharq_weight_sizes(256, 100, ok, ctypes.byref(wz)) == 1  # N % 128


def test_null_and_misaligned_pointers_rejected_before_any_launch(sq):
    cfg = sq.Config().c()
    act = sq.sharq_act(None, None, None, None, None, None, 16, 256, cfg)
    assert sq.sharq_prepare(ctypes.c_void_p(0x1000), sq.BF16, ctypes.byref(act), None) == 1
    p = ctypes.c_void_p
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5008), p(0x6000), 16, 256, cfg)
    assert sq.sharq_prepare(p(0x1000), sq.BF16, ctypes.byref(act), None) == 3  # rs misaligned
    w = sq.sharq_weight(p(0x1000), p(0x2000), p(0x3000), p(0x4000), 256, 128, cfg)
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000), 16, 512, cfg)
    assert sq.sharq_linear(ctypes.byref(act), ctypes.byref(w), p(0x7000), sq.BF16, None, 0,
                           None) == 1  # K mismatch
    assert sq.sharq_linear(ctypes.byref(act), ctypes.byref(w), p(0x7000), sq.F16, None, 0,
                           None) == 1  # bad out dtype


def test_prepare_rejects_tensors_beyond_32_bit_offsets(sq):
    p = ctypes.c_void_p
    cfg = sq.Config().c()
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000),
                       65536, 32768, cfg)
    assert sq.sharq_prepare(p(0x1000), sq.BF16, ctypes.byref(act), None) == 2


def test_prepare_rmsnorm_argument_checks(sq):
    p = ctypes.c_void_p
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000),
                       16, 256, sq.Config().c())
    f = sq.sharq_prepare_rmsnorm
    assert f(p(0x1000), None, 1e-6, sq.BF16, p(0x7000), ctypes.byref(act), None) == 1  # gamma
    assert f(p(0x1000), p(0x8000), 1e-6, sq.BF16, None, ctypes.byref(act), None) == 1  # rstd
    assert f(p(0x1000), p(0x8000), -1.0, sq.BF16, p(0x7000), ctypes.byref(act), None) == 1
    assert f(p(0x1000), p(0x8004), 1e-6, sq.BF16, p(0x7000), ctypes.byref(act), None) == 3
    elem = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000),
                        16, 256, sq.Config.from_names("nvfp4", "elem24").c())
    assert f(p(0x1000), p(0x8000), 1e-6, sq.BF16, p(0x7000), ctypes.byref(elem), None) == 2


def test_prepare_given_amax_and_alongside_argument_checks(sq):
    p = ctypes.c_void_p
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000),
                       16, 256, sq.Config().c())
    g = sq.sharq_prepare_given_amax
    assert g(p(0x1000), sq.BF16, None, ctypes.byref(act), None) == 1  # no amax
    assert g(p(0x1000), sq.BF16, p(0x7002), ctypes.byref(act), None) == 3  # misaligned amax
    for names in (("mxfp4", "pair48", True), ("nvfp4", "elem24", True), ("nvfp4", "none", False),
                  ("nvfp4", "pair48_given", True), ("nvfp4", "pair48", "own"),
                  ("nvfp4", "pair48", "unquantized")):
        other = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000),
                             16, 256, sq.Config.from_names(*names).c())
        assert g(p(0x1000), sq.BF16, p(0x7000), ctypes.byref(other), None) == 2, names
    a = sq.sharq_prepare_alongside
    assert a(None, sq.BF16, ctypes.byref(act), None) == 1
    assert a(p(0x1000), 7, ctypes.byref(act), None) == 1
    assert a(p(0x1008), sq.BF16, ctypes.byref(act), None) == 3


def test_wait_probe_argument_checks(sq):
    p = ctypes.c_void_p
    assert sq.sharq_wait_probe(None, 1, 10_000_000, None) == 1
    assert sq.sharq_wait_probe(p(0x1002), 1, 10_000_000, None) == 1  # misaligned
    assert sq.sharq_wait_probe(p(0x1000), 1, 1000, None) == 1        # limit below 1 ms
    assert sq.sharq_wait_probe(p(0x1000), 1, 20_000_000_000, None) == 1


def test_no_cpu_fallback_without_gpu(sq):
    """On a machine without a usable sm_100 GPU the compute calls return an error code
    (CUDA or ARCH) instead of computing anything on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    p = ctypes.c_void_p
    cfg = sq.Config().c()
    act = sq.sharq_act(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), p(0x6000), 16, 256, cfg)
    assert sq.sharq_prepare(p(0x1000), sq.BF16, ctypes.byref(act), None) in (4, 6)


def test_workspace_query_needs_a_device(sq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    n = ctypes.c_size_t(123)
    assert sq.sharq_linear_workspace_size(1, 4096, 14336, sq.Config().c(), ctypes.byref(n)) in (4, 6)
    assert sq.sharq_linear_workspace_size(1, 4096, 14336, sq.Config().c(), None) == 1
