"""Pins of the oracle's GEMM (brute-force triple loop, residual-off = sparse-only product)
and of its byte layouts (bijection and the positions fixed by the sm_100a MMA layouts)."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import layouts as L
from oracle import sharq as S
from workloads import heavy_activations


def _tiny(fmt, mask, M=3, K=256, N=4, seed=0):
    rng = np.random.default_rng(seed)
    x = heavy_activations(rng, M, K).values
    w = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    return S.prepare(x, fmt, mask), S.quantize_weight(w, fmt, mask)


@pytest.mark.parametrize("fmt", [S.NVFP4, S.MXFP4])
@pytest.mark.parametrize("mask", [S.PAIR48, S.ELEM24])
def test_linear_triple_loop(fmt, mask):
    """Y from the packed codes by a scalar loop, decoding each operand independently."""
    p, qw = _tiny(fmt, mask)
    M, K = p.keep.shape
    N = qw.wq.shape[0]
    Bb, Br, Bw = S.backbone_block(fmt, mask), S.residual_block(fmt), S.weight_block(fmt, mask)
    sval = F.e4m3_decode if fmt == S.NVFP4 else F.e8m0_decode

    def bval(m, k):
        if not p.keep[m, k]:
            return 0.0
        if mask == S.PAIR48:
            c = int(p.keep[m, :k].sum())  # compressed position of logical k
            return F.e2m1_decode(p.bq[m, c]) * sval(p.bs[m, c // 16])
        return F.e2m1_decode(p.bq[m, k]) * sval(p.bs[m, k // Bb])

    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                a = bval(m, k) + F.e2m1_decode(p.rq[m, k]) * sval(p.rs[m, k // Br])
                acc += a * F.e2m1_decode(qw.wq[n, k]) * sval(qw.ws[n, k // Bw])
            Y[m, n] = acc * float(p.s_g) * float(qw.s_gw)
    assert np.allclose(S.linear(p, qw), Y, rtol=1e-12, atol=1e-12)


def test_residual_off_equals_sparse_only():
    rng = np.random.default_rng(1)
    x = heavy_activations(rng, 8, 512).values
    w = rng.normal(0, 0.02, (512, 16)).astype(np.float32)
    qw = S.quantize_weight(w)
    p_off = S.prepare(x, residual=False)
    p_on = S.prepare(x)
    assert p_off.rq is None
    assert np.array_equal(S.linear(p_off, qw), S.linear_sparse_only(p_on, qw))


def test_row_col_sampling_is_exact():
    p, qw = _tiny(S.NVFP4, S.PAIR48, M=9, N=12)
    full = S.linear(p, qw)
    rows, cols = np.array([0, 4, 8]), np.array([1, 11])
    assert np.allclose(S.linear(p, qw, rows=rows, cols=cols), full[np.ix_(rows, cols)], rtol=1e-14)


def test_on_grid_input_has_zero_residual_and_plain_product():
    """x whose kept values sit on the FP4 grid and whose dropped values are 0: the residual
    codes are all zero and Y equals the plain product up to the float32 tensor scales."""
    x = np.zeros((1, 256), np.float32)
    x[0, 0:8] = [6, 6, 0, 0, 3, 3, 0, 0]  # pairs 0 and 2 kept; values on the grid
    w = np.zeros((256, 1), np.float32)
    w[0:8, 0] = [1, 1, 1, 1, 1, 1, 1, 1]
    p = S.prepare(x)
    qw = S.quantize_weight(w)
    assert np.all(p.rq == 0)
    assert np.isclose(S.linear(p, qw)[0, 0], 18.0, rtol=1e-6, atol=0)


# ----------------------------------------------------------------------------- layouts


def test_pack_nibbles_even_low():
    assert L.pack_nibbles(np.array([1, 2, 3, 4], np.uint8)).tolist() == [0x21, 0x43]
    c = np.random.default_rng(0).integers(0, 16, (5, 64)).astype(np.uint8)
    assert np.array_equal(L.unpack_nibbles(L.pack_nibbles(c)), c)


def test_scale_layout_positions():
    # positions fixed by the 128x4 scale-factor tile of the block-scaled MMA
    C = 8
    assert L.scale_offset(0, 0, C) == 0
    assert L.scale_offset(0, 1, C) == 1
    assert L.scale_offset(0, 3, C) == 3
    assert L.scale_offset(32, 0, C) == 4
    assert L.scale_offset(96, 2, C) == 14
    assert L.scale_offset(1, 0, C) == 16
    assert L.scale_offset(31, 3, C) == 31 * 16 + 3
    assert L.scale_offset(0, 4, C) == 512
    assert L.scale_offset(128, 0, C) == 1024
    assert L.scale_offset(129, 5, C) == 1024 + 512 + 16 + 1


@pytest.mark.parametrize("R,C", [(1, 1), (16, 16), (130, 9), (256, 448)])
def test_scale_layout_bijection(R, C):
    s = np.random.default_rng(1).integers(1, 255, (R, C)).astype(np.uint8)
    buf = L.to_scale_layout(s)
    assert buf.size == L.scale_layout_size(R, C)
    assert np.count_nonzero(buf) == R * C  # distinct positions, padding stays 0
    assert np.array_equal(L.from_scale_layout(buf, R, C), s)


def test_meta48_layout():
    M, K = 130, 512
    nib = np.random.default_rng(2).integers(0, 16, (M, K // 8)).astype(np.uint8)
    buf = L.to_meta48_layout(nib)
    assert buf.size == L.meta48_size(M, K)
    assert np.array_equal(L.from_meta48_layout(buf, M, K), nib)
    # row r, group g (< 32) of the first 256-K slice -> byte 16 r + g // 2
    assert buf[16 * 5 + 3] == (nib[5, 6] | (nib[5, 7] << 4))
    # second slice starts after all padded rows of the first one
    assert buf[256 * 16 + 16 * 2] == (nib[2, 32] | (nib[2, 33] << 4))
    # padding rows carry the valid pattern "pairs 0 and 1"
    assert np.all(buf[16 * 130: 16 * 256] == 0x44)
