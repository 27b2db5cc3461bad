"""The no-allocation linear entry point, checked against sharq_linear.

sharq_linear_noalloc is for callers that cannot allocate device memory (code captured into
CUDA graphs, allocator-free runtimes, hosts that forbid allocation on the hot path): the
split-K scratch it needs for decode-sized M is a fixed array inside the library instead of
a caller workspace. These tests call it through the C ABI, two calls in a row, and compare
each result with sharq_linear given a caller-owned workspace, and, on two shapes, with the
oracle's product, within the FP32 tolerance of the other GEMM tests. This file is collected last so that a failure here cannot hide an
earlier one."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5  # relative Frobenius error, as in the other GEMM parity tests


def _setup(M, K, N):
    import torch

    import fp4_sparse_dense_b200 as sq
    from workloads import gaussian_weight, heavy_activations, to_device
    rng = np.random.default_rng(M + K + N)
    x = heavy_activations(rng, M, K, per_row=True)
    w = gaussian_weight(rng, K, N)
    cfg = sq.Config()
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    return sq, torch, act, wt


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm())


@pytest.mark.parametrize("M,K,N", [(1, 14336, 4096), (16, 14336, 4096), (64, 14336, 4096),
                                   (8, 4096, 1024)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_noalloc_matches_linear_on_two_calls(M, K, N, out):
    sq, torch, act, wt = _setup(M, K, N)
    dt, code = (torch.float32, sq.F32) if out == "f32" else (torch.bfloat16, sq.BF16)
    ws = sq.linear_workspace(M, N, K, act.cfg)
    assert ws is not None  # these shapes run the split-K path, i.e. use scratch memory
    ref = sq.linear(act, wt, out_dtype=dt, workspace=ws)
    ca, cw = act.c(), wt.c()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
        rc = sq.sharq_linear_noalloc(ctypes.byref(ca), ctypes.byref(cw),
                                     ctypes.c_void_p(y.data_ptr()), code, stream)
        assert rc == 0, sq.sharq_status_string(rc)
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        assert not torch.isnan(y).any()
        tol = TOL_F32 if out == "f32" else 1e-3
        assert _rel(y, ref) <= tol


@pytest.mark.parametrize("M,K,N", [(8, 4096, 1024), (16, 14336, 4096)])
def test_noalloc_matches_oracle(M, K, N):
    """The same calls against the oracle: its float64 product of the dequantised operands,
    FP32 output held to the GEMM parity tests' 1e-5 relative Frobenius error."""
    from oracle import sharq as S
    from workloads import gaussian_weight, heavy_activations, to_device
    import torch

    import fp4_sparse_dense_b200 as sq
    rng = np.random.default_rng(7 * M + K + N)
    x = heavy_activations(rng, M, K, per_row=True)
    w = gaussian_weight(rng, K, N)
    cfg = sq.Config()
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    assert sq.linear_workspace(M, N, K, cfg) is not None  # the split-K path: library scratch
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ca, cw = act.c(), wt.c()
    rc = sq.sharq_linear_noalloc(ctypes.byref(ca), ctypes.byref(cw),
                                 ctypes.c_void_p(y.data_ptr()), sq.F32,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, sq.sharq_status_string(rc)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    y64 = S.linear(S.prepare(x.values), S.quantize_weight(w.values))
    got = y.cpu().numpy().astype(np.float64)
    assert float(np.linalg.norm(got - y64) / np.linalg.norm(y64)) <= TOL_F32


def test_noalloc_unsplit_shape_matches_linear():
    sq, torch, act, wt = _setup(512, 1024, 512)
    assert sq.linear_workspace(512, 512, 1024, act.cfg) is None
    ref = sq.linear(act, wt, out_dtype=torch.float32, workspace=None)
    y = torch.empty(512, 512, dtype=torch.float32, device="cuda")
    ca, cw = act.c(), wt.c()
    rc = sq.sharq_linear_noalloc(ctypes.byref(ca), ctypes.byref(cw),
                                 ctypes.c_void_p(y.data_ptr()), sq.F32,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert _rel(y, ref) <= TOL_F32


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """M=128, K=2048, N=8448 splits K four ways: 4 x 128 x 8448 x 4 bytes > 16 MiB."""
    sq, torch, act, wt = _setup(128, 2048, 8448)
    n = ctypes.c_size_t(0)
    assert sq.sharq_linear_workspace_size(128, 8448, 2048, act.cfg.c(), ctypes.byref(n)) == 0
    assert n.value > 16 << 20
    y = torch.empty(128, 8448, dtype=torch.bfloat16, device="cuda")
    ca, cw = act.c(), wt.c()
    rc = sq.sharq_linear_noalloc(ctypes.byref(ca), ctypes.byref(cw),
                                 ctypes.c_void_p(y.data_ptr()), sq.BF16,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 2  # SHARQ_ERR_UNSUPPORTED, nothing launched
