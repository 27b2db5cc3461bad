"""GPU parity of the offline weight quantisation: one FP4 code payload (K-major) and both
scale views, bit-exact against the CPU oracle."""
import numpy as np
import pytest

from oracle import sharq as S
from tests.gpu_helpers import assert_bytes_equal, cfg_of, to_device, weight_bytes
from workloads import BF16, F16, gaussian_weight

pytestmark = pytest.mark.gpu


def run_wq(w16, fmt, mask):
    import fp4_sparse_dense_b200 as sq
    import torch
    qw = sq.quantize_weight(to_device(w16), cfg_of(fmt, mask))
    torch.cuda.synchronize()
    return qw


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("mask", ["pair48", "elem24"])
@pytest.mark.parametrize("K,N,dtype", [(256, 128, F16), (512, 384, BF16), (1024, 256, BF16),
                                       (4096, 1024, BF16)])
def test_weight_quant_bit_exact(fmt, mask, K, N, dtype):
    w = gaussian_weight(np.random.default_rng(K + N), K, N, dtype)
    got = weight_bytes(run_wq(w, fmt, mask))
    want = S.weight_buffers(S.quantize_weight(w.values, fmt, mask))
    assert_bytes_equal(got, want)


def test_weight_quant_full_size_sampled_columns():
    """W[4096 x 14336]: tensor scale exact; 64 sampled output rows bit-exact."""
    from oracle import layouts as L
    K, N = 4096, 14336
    rng = np.random.default_rng(5)
    w = gaussian_weight(rng, K, N)
    got = weight_bytes(run_wq(w, "nvfp4", "pair48"))
    amax = S.amax_of(w.values)
    assert got["tensor_scale"][0] == S.tensor_scales(amax)[0]
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 62, replace=False)]))
    q = S.quantize_weight(w.values[:, cols], "nvfp4", "pair48", amax=amax)
    codes = got["codes"].reshape(N, K // 2)[cols]
    assert np.array_equal(codes, L.pack_nibbles(q.wq))
    assert np.array_equal(L.from_scale_layout(got["scales_sparse"], N, K // 32)[cols], q.ws)
    assert np.array_equal(L.from_scale_layout(got["scales_dense"], N, K // 16)[cols],
                          S.weight_scale_view(q, 16))
