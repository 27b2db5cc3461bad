"""GPU parity of the preparation with a caller-supplied NVFP4 tensor amax
(sharq_prepare_given_amax: one kernel, the mask computed in it): every byte equal to the
oracle's prepare(..., amax=value), for the tensor's own amax, a larger one, and a smaller
one under which large values saturate; and the GEMM over it."""
import numpy as np
import pytest

from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, cfg_of, rel_fro, to_device
from workloads import BF16, F16, gaussian_weight, heavy_activations

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,dtype", [(1, 256, BF16), (127, 512, F16), (300, 1024, BF16),
                                       (2048, 4096, BF16)])
@pytest.mark.parametrize("scale", [1.0, 3.0, 0.25])
def test_given_amax_bit_exact(residual, M, K, dtype, scale):
    import fp4_sparse_dense_b200 as sq
    import torch
    x = heavy_activations(np.random.default_rng(M + K + int(scale * 8)), M, K, dtype=dtype)
    amax = np.float32(S.amax_of(x.values) * np.float32(scale))
    cfg = cfg_of("nvfp4", "pair48", residual)
    act = sq.prepare(to_device(x), cfg, amax=torch.tensor([amax], dtype=torch.float32).cuda())
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    want = S.act_buffers(S.prepare(x.values, "nvfp4", "pair48", residual=residual, amax=amax))
    assert_bytes_equal(act_bytes(act), want)
    assert float(act.tensor_scale[1]) == float(amax)


def test_given_amax_linear_and_rejected_configs():
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K, N = 512, 2048, 1024
    rng = np.random.default_rng(77)
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    amax = np.float32(S.amax_of(x.values))
    cfg = cfg_of("nvfp4", "pair48")
    a_t = torch.tensor([amax], dtype=torch.float32).cuda()
    act = sq.prepare(to_device(x), cfg, amax=a_t)
    ref = sq.prepare(to_device(x), cfg)  # the in-call amax is the same value here
    qw = sq.quantize_weight(to_device(w), cfg)
    y = sq.linear(act, qw, out_dtype=torch.float32)
    y_ref = sq.linear(ref, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    assert torch.equal(y, y_ref)
    y64 = S.linear(S.prepare(x.values, amax=amax), S.quantize_weight(w.values))
    assert rel_fro(y.double().cpu().numpy(), y64) <= 1e-5
    for c in (cfg_of("mxfp4", "pair48"), cfg_of("nvfp4", "elem24"), cfg_of("nvfp4", "pair48", "own")):
        with pytest.raises(sq.SharqError):
            sq.prepare(to_device(x), c, amax=a_t)
