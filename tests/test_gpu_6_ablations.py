"""GPU parity of the ablation modes against the oracle: the residual against the
unquantised backbone, a caller-supplied (static) pair mask, and plain FP4 without a mask.
Prepared bytes bit-exact; the linear layer in FP32 output within the parity tolerance."""
import numpy as np
import pytest

from oracle import layouts as L
from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, cfg_of, rel_fro, to_device
from workloads import gaussian_weight, heavy_activations

pytestmark = pytest.mark.gpu

SHAPES = [(1, 256, 128), (127, 512, 256), (300, 1024, 384)]


def _inputs(M, K, N, seed):
    rng = np.random.default_rng(seed)
    return heavy_activations(rng, M, K, per_row=True), gaussian_weight(rng, K, N)


def _linear_f32(act, wt):
    import fp4_sparse_dense_b200 as sq
    import torch
    y = sq.linear(act, wt, out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    return y


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("mask", ["pair48", "elem24"])
@pytest.mark.parametrize("M,K,N", SHAPES)
def test_residual_against_unquantized_backbone(fmt, mask, M, K, N):
    import fp4_sparse_dense_b200 as sq
    x, w = _inputs(M, K, N, M + K)
    cfg = cfg_of(fmt, mask, "unquantized")
    act = sq.prepare(to_device(x), cfg)
    p = S.prepare(x.values, fmt, mask, residual_ref="unquantized")
    assert_bytes_equal(act_bytes(act), S.act_buffers(p))
    wt = sq.quantize_weight(to_device(w), cfg)
    y64 = S.linear(p, S.quantize_weight(w.values, fmt, mask))
    assert rel_fro(_linear_f32(act, wt), y64) <= 1e-5


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,N", SHAPES)
def test_static_mask_supplied_by_the_caller(fmt, residual, M, K, N):
    """Static mask from a calibration tensor's per-column max |x|, written into bm in the
    PAIR metadata layout before the call; the kernels must keep it and use it."""
    import fp4_sparse_dense_b200 as sq
    import torch
    x, w = _inputs(M, K, N, 3 * M + K)
    calib = heavy_activations(np.random.default_rng(99), 64, K, per_row=True)
    given = S.static_keep_pairs48(calib.values, M)
    p = S.prepare(x.values, fmt, S.PAIR48_GIVEN, residual=residual, given=given)
    cfg = cfg_of(fmt, "pair48_given", residual)
    act = sq.empty_act(M, K, cfg)
    bm = S.act_buffers(p)["bm"]
    act.bm[: bm.size].copy_(torch.from_numpy(np.ascontiguousarray(bm)).cuda())
    sq.prepare(to_device(x), cfg, out=act)
    assert_bytes_equal(act_bytes(act), S.act_buffers(p))
    wt = sq.quantize_weight(to_device(w), cfg)
    y64 = S.linear(p, S.quantize_weight(w.values, fmt, S.PAIR48_GIVEN))
    assert rel_fro(_linear_f32(act, wt), y64) <= 1e-5


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,N", SHAPES)
def test_plain_fp4_without_mask(fmt, residual, M, K, N):
    import fp4_sparse_dense_b200 as sq
    x, w = _inputs(M, K, N, 5 * M + K)
    cfg = cfg_of(fmt, "none", residual)
    act = sq.prepare(to_device(x), cfg)
    assert act.bm is None
    p = S.prepare(x.values, fmt, S.NONE, residual=residual)
    assert_bytes_equal(act_bytes(act), S.act_buffers(p))
    wt = sq.quantize_weight(to_device(w), cfg)
    y64 = S.linear(p, S.quantize_weight(w.values, fmt, S.NONE))
    assert rel_fro(_linear_f32(act, wt), y64) <= 1e-5
