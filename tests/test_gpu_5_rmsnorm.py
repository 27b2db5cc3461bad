"""GPU parity of the preparation with RMSNorm absorbed (sharq_prepare_rmsnorm) against the
CPU oracle (oracle/norm.py + oracle/sharq.py): per-row rstd and every prepared byte
bit-exact, across formats, dtypes, residual on/off and ragged row counts; repeated calls
into one buffer; and the linear layer on the normalised input at a benchmark shape."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import norm as N
from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, cfg_of, rel_fro, to_device
from workloads import BF16, F16, Tensor16, gaussian_weight, heavy_activations, to_dtype

pytestmark = pytest.mark.gpu


def _gamma(rng, K, dtype):
    """Norm weights around 1 with a few negative and large entries."""
    g = rng.normal(1.0, 0.3, K).astype(np.float32)
    g[rng.choice(K, max(1, K // 64), replace=False)] *= -3.0
    v, b = to_dtype(g, dtype)
    return Tensor16(v, b, dtype)


def _run(x16, g16, eps, fmt, residual=True):
    import fp4_sparse_dense_b200 as sq
    import torch
    act, rstd = sq.prepare_rmsnorm(to_device(x16), to_device(g16), eps,
                                   cfg_of(fmt, "pair48", residual))
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    return act, rstd.cpu().numpy()


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,dtype", [(1, 256, BF16), (16, 256, F16), (127, 512, BF16),
                                       (300, 4096, BF16), (513, 2048, F16)])
def test_rmsnorm_prep_bit_exact(fmt, residual, M, K, dtype):
    rng = np.random.default_rng(M * 11 + K)
    x = heavy_activations(rng, M, K, dtype=dtype)
    g = _gamma(rng, K, dtype)
    eps = 1e-5
    act, rstd = _run(x, g, eps, fmt, residual)
    p, y, rstd_want = N.prepare_rmsnorm(x.values, g.values, eps, dtype, fmt, "pair48",
                                        residual=residual)
    assert np.array_equal(rstd.view(np.uint32), rstd_want.view(np.uint32))
    assert_bytes_equal(act_bytes(act), S.act_buffers(p))


def test_rmsnorm_prep_repeated_calls_on_one_buffer():
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K = 200, 1024
    cfg = cfg_of("nvfp4", "pair48")
    act = sq.empty_act(M, K, cfg)
    rng = np.random.default_rng(9)
    for scale, eps in ((1.0, 1e-6), (1e-3, 1e-6), (50.0, 0.5), (1.0, 0.0)):
        v, b = to_dtype(heavy_activations(rng, M, K).values * np.float32(scale), BF16)
        x = Tensor16(v, b, BF16)
        g = _gamma(rng, K, BF16)
        sq.prepare_rmsnorm(to_device(x), to_device(g), eps, cfg, out=act)
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        p, y, _ = N.prepare_rmsnorm(x.values, g.values, eps, BF16)
        assert_bytes_equal(act_bytes(act), S.act_buffers(p))


def test_rmsnorm_linear_full_size_sampled():
    """mlp_gate_up shape with the norm absorbed: sampled rows and columns of Y against the
    oracle's FP64 product on the normalised, prepared rows."""
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K, N_ = 4096, 4096, 14336
    rng = np.random.default_rng(77)
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N_)
    g = _gamma(rng, K, BF16)
    cfg = cfg_of("nvfp4", "pair48")
    act, rstd = sq.prepare_rmsnorm(to_device(x), to_device(g), 1e-6, cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    y = sq.linear(act, wt).float().cpu().numpy()
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    yn, rstd_want = N.rmsnorm(x.values, g.values, 1e-6, BF16)
    assert np.array_equal(rstd.cpu().numpy(), rstd_want)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 24, replace=False)]))
    cols = np.unique(np.concatenate([[0, N_ - 1], rng.choice(N_, 160, replace=False)]))
    p = S.prepare(yn[rows], amax=S.amax_of(yn))
    qw = S.quantize_weight(w.values[:, cols], amax=S.amax_of(w.values))
    assert rel_fro(y[np.ix_(rows, cols)], F.bf16_round(S.linear(p, qw))) <= 1e-3
