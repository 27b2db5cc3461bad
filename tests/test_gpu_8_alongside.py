"""GPU parity of the preparation launched to share the GPU with a GEMM
(sharq_prepare_alongside): the same bytes as the oracle on ragged shapes, also while a
GEMM runs on another stream, and the tensor-amax hand-over when it alternates with the
ordinary launch on one activation buffer."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, cfg_of, rel_fro, to_device
from workloads import BF16, F16, gaussian_weight, heavy_activations

pytestmark = pytest.mark.gpu


def prep(x16, cfg, alongside, out=None, stream=None):
    import fp4_sparse_dense_b200 as sq
    return sq.prepare(to_device(x16), cfg, out=out, stream=stream, alongside=alongside)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("mask", ["pair48", "elem24"])
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,dtype", [(1, 256, BF16), (127, 512, F16), (513, 2048, BF16),
                                       (2048, 4096, BF16)])
def test_alongside_bit_exact(fmt, mask, residual, M, K, dtype):
    import fp4_sparse_dense_b200 as sq
    import torch
    x = heavy_activations(np.random.default_rng(M + 3 * K), M, K, dtype=dtype)
    act = prep(x, cfg_of(fmt, mask, residual), alongside=True)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    want = S.act_buffers(S.prepare(x.values, fmt, mask, residual=residual))
    assert_bytes_equal(act_bytes(act), want)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_alongside_beside_a_running_gemm(fmt):
    """Batch b's preparation on a side stream while batch a's GEMM runs on the main stream:
    b's bytes equal the oracle's and a's output equals the same GEMM run alone."""
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K, N = 1024, 2048, 4096
    rng = np.random.default_rng(81)
    xa = heavy_activations(rng, M, K)
    xb = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of(fmt, "pair48", True)
    Wd = to_device(w)
    qw = sq.quantize_weight(Wd, cfg)
    act_a = sq.prepare(to_device(xa), cfg)
    y_alone = sq.linear(act_a, qw)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    Xb = to_device(xb)
    act_b = sq.empty_act(M, K, cfg)
    side.wait_stream(main)
    ys = []
    for _ in range(4):  # several GEMMs back to back, so that the preparation lands among them
        ys.append(sq.linear(act_a, qw))
    with torch.cuda.stream(side):
        sq.prepare(Xb, cfg, out=act_b, stream=side, alongside=True)
    main.wait_stream(side)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    want = S.act_buffers(S.prepare(xb.values, fmt, "pair48"))
    assert_bytes_equal(act_bytes(act_b), want)
    for y in ys:
        assert torch.equal(y, y_alone)
    # and batch b's product through the GEMM matches the oracle
    y_b = sq.linear(act_b, qw, out_dtype=torch.float32).double().cpu().numpy()
    y64 = S.linear(S.prepare(xb.values, fmt, "pair48"), S.quantize_weight(w.values, fmt, "pair48"))
    assert rel_fro(y_b, y64) <= 1e-5


def test_alongside_and_ordinary_launch_alternate_on_one_buffer():
    """The NVFP4 tensor amax is handed from the first kernel to the second through the
    activation's state words; launches of different grid sizes alternate on them."""
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K = 384, 1024
    cfg = cfg_of("nvfp4", "pair48", True)
    act = sq.empty_act(M, K, cfg)
    for i in range(6):
        x = heavy_activations(np.random.default_rng(100 + i), M, K, dtype=F16 if i % 3 else BF16)
        prep(x, cfg, alongside=bool(i % 2), out=act)
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        assert_bytes_equal(act_bytes(act), S.act_buffers(S.prepare(x.values, "nvfp4", "pair48")))
        assert float(act.tensor_scale[2]) == 0.0 and float(act.tensor_scale[3]) == 0.0
