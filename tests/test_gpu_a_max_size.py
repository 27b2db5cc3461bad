"""The largest tensor the pair-mask preparation accepts (M * K just below 2^31 elements: its
kernels address X and their outputs with 32-bit offsets) and a GEMM over it: sampled rows
bit-exact against the oracle, the first and last rows included, and Y on those rows within
the GEMM tolerances. X is drawn on the device (seeded) with |x| <= 30 everywhere and one
planted element of 100, so the tensor amax is known without reading 4 GB back."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import layouts as L
from oracle import sharq as S
from tests.gpu_helpers import rel_fro, to_device
from workloads import gaussian_weight

pytestmark = pytest.mark.gpu

M, K, N = 131071, 16384, 128  # M * K = 2^31 - 16384
PLANT = (77777, 12345)


def _rows_of_scale_layout(dev_buf, rows, cols):
    """Canonical scale bytes of `rows` from a tiled scale buffer on the device, copying
    only the 128-row tiles that hold them."""
    chunk = (cols // 4) * 512
    out = []
    for r in rows:
        rb = r // 128
        tile = dev_buf[rb * chunk:(rb + 1) * chunk].cpu().numpy()
        out.append(L.from_scale_layout(tile, 128, cols)[r % 128])
    return np.stack(out)


def _rows_of_meta48(dev_buf, rows, Mp):
    out = []
    for r in rows:
        rb = r // 128
        parts = [dev_buf[q * Mp * 16 + rb * 2048:q * Mp * 16 + (rb + 1) * 2048].cpu().numpy()
                 for q in range(K // 256)]
        out.append(L.from_meta48_layout(np.concatenate(parts), 128, K)[r % 128])
    return np.stack(out)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_largest_accepted_tensor_prepare_and_linear(fmt):
    import fp4_sparse_dense_b200 as sq
    import torch
    g = torch.Generator(device="cuda").manual_seed(2024)
    X = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, M, 8192):
        r1 = min(M, r0 + 8192)
        X[r0:r1] = (torch.randn(r1 - r0, K, generator=g, device="cuda") * 3).clamp_(-30, 30)
    X[PLANT] = 100.0
    cfg = sq.Config.from_names(fmt, "pair48", True)
    act = sq.prepare(X, cfg)
    rng = np.random.default_rng(9)
    w = gaussian_weight(rng, K, N)
    qw = sq.quantize_weight(to_device(w), cfg)
    y = sq.linear(act, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0

    amax = np.float32(100.0) if fmt == "nvfp4" else None
    if fmt == "nvfp4":
        assert float(act.tensor_scale[0]) == S.tensor_scales(amax)[0]
    rows = np.unique(np.concatenate([[0, 1, PLANT[0], M - 2, M - 1],
                                     rng.choice(M, 6, replace=False)]))
    xs = X[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    p = S.prepare(xs, fmt, "pair48", amax=amax)
    bq = act.bq.view(M, K // 4)[torch.from_numpy(rows).cuda()].cpu().numpy()
    rq = act.rq.view(M, K // 2)[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(bq, L.pack_nibbles(p.bq))
    assert np.array_equal(rq, L.pack_nibbles(p.rq))
    assert np.array_equal(_rows_of_scale_layout(act.bs, rows, K // 32), p.bs)
    assert np.array_equal(_rows_of_scale_layout(act.rs, rows, K // S.residual_block(fmt)), p.rs)
    assert np.array_equal(_rows_of_meta48(act.bm, rows, (M + 127) // 128 * 128), p.meta)

    y64 = S.linear(p, S.quantize_weight(w.values, fmt, "pair48"))
    ys = y[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    assert rel_fro(ys, y64) <= 1e-5
