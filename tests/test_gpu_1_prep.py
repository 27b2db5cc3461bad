"""GPU parity of the activation preparation (amax pass + fused prep kernel) against the
CPU oracle: masks, FP4 codes, scales, metadata and the tensor scale bit-exact, across
formats, masks, dtypes, ragged row counts and the benchmark shapes."""
import numpy as np
import pytest

from oracle import sharq as S
from tests.gpu_helpers import (act_bytes, assert_bytes_equal, cfg_of, sampled_act_rows,
                               to_device)
from workloads import BF16, F16, Tensor16, heavy_activations, tiny_activations, to_dtype

pytestmark = pytest.mark.gpu

FMTS = ["nvfp4", "mxfp4"]
MASKS = ["pair48", "elem24"]


def run_prep(x16, fmt, mask, residual=True):
    import fp4_sparse_dense_b200 as sq
    import torch
    act = sq.prepare(to_device(x16), cfg_of(fmt, mask, residual))
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    return act


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mask", MASKS)
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,K,dtype", [(1, 256, BF16), (16, 256, F16), (127, 512, BF16),
                                       (128, 1024, BF16), (300, 768, F16), (513, 2048, BF16)])
def test_prep_bit_exact(fmt, mask, residual, M, K, dtype):
    rng = np.random.default_rng(M * 7 + K)
    x = heavy_activations(rng, M, K, dtype=dtype)
    got = act_bytes(run_prep(x, fmt, mask, residual))
    want = S.act_buffers(S.prepare(x.values, fmt, mask, residual=residual))
    assert_bytes_equal(got, want)


def test_prep_tiny_config_fp16_elem24():
    x = tiny_activations()  # X[16x256] fp16, 4 outlier channels x30
    got = act_bytes(run_prep(x, "nvfp4", "elem24"))
    want = S.act_buffers(S.prepare(x.values, "nvfp4", "elem24"))
    assert_bytes_equal(got, want)


def test_prep_worked_example():
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "worked_block_nvfp4_pair48.json")))
    xv = np.zeros((1, 256), np.float32)
    xv[0, :32] = g["x_first32"]
    v, b = to_dtype(xv, BF16)
    got = act_bytes(run_prep(Tensor16(v, b, BF16), "nvfp4", "pair48"))
    want = S.act_buffers(S.prepare(v, "nvfp4", "pair48"))
    assert_bytes_equal(got, want)
    assert got["tensor_scale"][0] == 1.0


@pytest.mark.parametrize("special", ["zeros", "ties", "negzero", "subnormal", "huge"])
def test_prep_edge_values(special):
    M, K = 64, 512
    rng = np.random.default_rng(3)
    if special == "zeros":
        xv = np.zeros((M, K), np.float32)
    elif special == "ties":
        xv = rng.integers(-2, 3, (M, K)).astype(np.float32)
    elif special == "negzero":
        xv = np.where(rng.random((M, K)) < 0.5, -0.0, 1e-3).astype(np.float32)
        xv[:, ::17] = -3.0
    elif special == "subnormal":
        xv = (rng.standard_normal((M, K)) * 1e-39).astype(np.float32)
        xv[0, 0] = 1.0
    else:
        xv = (rng.standard_normal((M, K)) * 1e30).astype(np.float32)
    for fmt in FMTS:
        for mask in MASKS:
            v, b = to_dtype(xv, BF16)
            got = act_bytes(run_prep(Tensor16(v, b, BF16), fmt, mask))
            want = S.act_buffers(S.prepare(v, fmt, mask))
            assert_bytes_equal(got, want)


@pytest.mark.parametrize("name,M,K,per_row", [("attn_proj", 2048, 4096, False),
                                               ("mlp_gate_up", 4096, 4096, False),
                                               ("mlp_down", 4096, 14336, True)])
def test_prep_full_size_sampled_rows(name, M, K, per_row):
    """Benchmark shapes: tensor scale exact, and 48 sampled rows (first, last, random)
    bit-exact against the oracle run on those rows with the whole tensor's scale."""
    rng = np.random.default_rng(11)
    x = heavy_activations(rng, M, K, per_row=per_row)
    act = run_prep(x, "nvfp4", "pair48")
    got = act_bytes(act)
    amax = S.amax_of(x.values)
    assert got["tensor_scale"][0] == S.tensor_scales(amax)[0]
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 46, replace=False)]))
    g = sampled_act_rows(got, rows, M, K, "nvfp4", "pair48")
    p = S.prepare(x.values[rows], "nvfp4", "pair48", amax=amax)
    from oracle import layouts as L
    assert np.array_equal(g["bq"], L.pack_nibbles(p.bq))
    assert np.array_equal(g["bs"], p.bs)
    assert np.array_equal(g["meta"], p.meta)
    assert np.array_equal(g["rq"], L.pack_nibbles(p.rq))
    assert np.array_equal(g["rs"], p.rs)


@pytest.mark.parametrize("mask", MASKS)
def test_prep_repeated_calls_on_one_buffer(mask):
    """The tensor amax is reduced afresh on every call into the same buffers: a small X after
    a large one gets its own (smaller) tensor scale, and the outputs of every call match the
    oracle. With the pair mask this also walks the in-kernel reduction state through
    several generations."""
    import fp4_sparse_dense_b200 as sq
    import torch
    M, K = 300, 1024
    cfg = cfg_of("nvfp4", mask)
    act = sq.empty_act(M, K, cfg)
    rng = np.random.default_rng(5)
    for scale in (1.0, 1e-3, 40.0, 0.5, 0.5):
        x = heavy_activations(rng, M, K)
        v, b = to_dtype(x.values * np.float32(scale), BF16)
        x = Tensor16(v, b, BF16)
        sq.prepare(to_device(x), cfg, out=act)
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        got = act_bytes(act)
        want = S.act_buffers(S.prepare(x.values, "nvfp4", mask))
        assert_bytes_equal(got, want)
        assert float(act.tensor_scale[1].item()) == float(np.abs(x.values).max())
