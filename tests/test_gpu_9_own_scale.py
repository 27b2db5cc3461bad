"""GPU parity of the variant whose residual has its own tensor scale (s_r = amax|r| / 2688
instead of sharing s_g; the alternative the page's decomposition leaves open, here with two
FP32 accumulators, Y = s_gw * (s_g * acc_backbone + s_r * acc_residual)): codes, scales,
metadata and both tensor scales bit-exact against the oracle's prepare(...,
residual_scale="own"), and Y against the oracle's float64 product of the same dequantised
operands (float32 output within 1e-5, bf16 output within 1e-3 of bf16(Y64), the tolerances
of the method's own GEMM test)."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, cfg_of, rel_fro, to_device
from workloads import BF16, F16, gaussian_weight, heavy_activations

pytestmark = pytest.mark.gpu


def gpu_prepare(x16, mask="pair48", given=None):
    import fp4_sparse_dense_b200 as sq
    import torch
    cfg = cfg_of("nvfp4", mask, "own")
    act = sq.empty_act(*x16.values.shape, cfg)
    if given is not None:
        from oracle import layouts as L
        meta = S.canonical_metadata(x16.values, S.PAIR48_GIVEN, given)
        bm = torch.from_numpy(np.ascontiguousarray(L.to_meta48_layout(meta))).cuda()
        act.bm[: bm.numel()].copy_(bm)
    sq.prepare(to_device(x16), cfg, out=act)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    return act


def check_prep(act, p):
    assert_bytes_equal(act_bytes(act), S.act_buffers(p))
    ts = act.tensor_scale.cpu().numpy()
    assert ts[6] == np.float32(p.s_r)
    assert ts[7] == np.float32(np.max(np.abs(p.r)))
    assert np.all(ts[2:6] == 0)  # both amax states handed back for the next call


@pytest.mark.parametrize("M,K,dtype", [(1, 256, BF16), (127, 512, F16), (300, 1024, BF16),
                                       (513, 2048, BF16), (2048, 4096, BF16)])
def test_own_scale_prep_bit_exact(M, K, dtype):
    x = heavy_activations(np.random.default_rng(7 * M + K), M, K, dtype=dtype)
    check_prep(gpu_prepare(x), S.prepare(x.values, "nvfp4", "pair48", residual_scale="own"))


def test_own_scale_prep_with_a_given_mask():
    M, K = 200, 1024
    x = heavy_activations(np.random.default_rng(5), M, K)
    given = S.static_keep_pairs48(x.values, M)
    check_prep(gpu_prepare(x, "pair48_given", given),
               S.prepare(x.values, "nvfp4", S.PAIR48_GIVEN, given=given, residual_scale="own"))


def test_own_scale_repeated_calls_on_one_buffer():
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K = 256, 512
    cfg = cfg_of("nvfp4", "pair48", "own")
    act = sq.empty_act(M, K, cfg)
    for i in range(4):
        x = heavy_activations(np.random.default_rng(40 + i), M, K)
        sq.prepare(to_device(x), cfg, out=act)
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        check_prep(act, S.prepare(x.values, "nvfp4", "pair48", residual_scale="own"))


@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (100, 1024, 384), (300, 2048, 256),
                                   (1024, 4096, 4096)])
@pytest.mark.parametrize("out_f32", [True, False])
def test_own_scale_linear(M, K, N, out_f32):
    import fp4_sparse_dense_b200 as sq
    import torch
    rng = np.random.default_rng(M + K + N)
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of("nvfp4", "pair48", "own")
    act = gpu_prepare(x)
    qw = sq.quantize_weight(to_device(w), cfg)
    y = sq.linear(act, qw, out_dtype=torch.float32 if out_f32 else torch.bfloat16)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    y = y.float().cpu().numpy().astype(np.float64)
    p = S.prepare(x.values, "nvfp4", "pair48", residual_scale="own")
    y64 = S.linear(p, S.quantize_weight(w.values, "nvfp4", "pair48"))
    if out_f32:
        assert rel_fro(y, y64) <= 1e-5
    else:
        assert rel_fro(y, F.bf16_round(y64)) <= 1e-3
