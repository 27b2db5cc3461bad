"""Pins of the oracle's SharQ decomposition: the hand-worked example, brute force on tiny
inputs, and the invariants the SharQ page states (pith.science 2606.26587, "Core claim":
backbone = largest-|x| entries under an N:M mask; residual defined against the
*quantised* backbone; the dense path compensates mask loss and backbone quantisation
error)."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import formats as F
from oracle import sharq as S
from workloads import heavy_activations

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_block_nvfp4_pair48.json")


def _worked_x():
    g = json.load(open(GOLD))
    x = np.zeros((1, 256), np.float32)
    x[0, :32] = g["x_first32"]
    return g, x


def test_worked_example_nvfp4():
    g, x = _worked_x()
    p = S.prepare(x, S.NVFP4, S.PAIR48)
    e = g["nvfp4"]
    assert p.s_g == np.float32(e["s_g"])
    assert list(p.meta[0, :4]) == e["meta_first4"]
    assert np.all(p.meta[0, 4:] == e["meta_rest"])
    assert list(p.bq[0, :16]) == e["bq_block0"]
    assert np.all(p.bq[0, 16:] == 0)
    assert list(p.bs[0]) == e["bs"]
    assert list(p.rq[0, :32]) == e["rq_first32"]
    assert np.all(p.rq[0, 32:] == 0)
    assert list(p.rs[0]) == e["rs"]


def test_worked_example_mxfp4():
    g, x = _worked_x()
    p = S.prepare(x, S.MXFP4, S.PAIR48)
    e = g["mxfp4"]
    assert list(p.bq[0, :16]) == e["bq_block0"]
    assert p.bs[0, 0] == e["bs_first"]
    assert p.r[0, 0] == e["r0"]
    assert list(p.rq[0, :32]) == e["rq_first32"]
    assert p.rs[0, 0] == e["rs_first"]


GOLD_SG = os.path.join(os.path.dirname(__file__), "golden", "worked_block_nvfp4_sg_not_one.json")
GOLD_W = os.path.join(os.path.dirname(__file__), "golden", "worked_weight_k64_n2.json")


def test_worked_example_tensor_scale_not_one():
    """s_g = float32(1.75 / 2688) != 1: the block scale comes from a * (448 / amax), where a
    block max of 0.71875 lands exactly on an E4M3 tie (184 -> 192, code 0x74); the order
    (a / 6) / s_g would give 0x73 (hand-worked fixture)."""
    g = json.load(open(GOLD_SG))
    x = np.zeros((1, 256), np.float32)
    for k, v in g["x_nonzero"].items():
        x[0, int(k)] = v
    p = S.prepare(x, S.NVFP4, S.PAIR48)
    e = g["expected"]
    assert np.float32(p.s_g).view(np.uint32) == int(e["s_g_bits"], 16)
    assert np.all(p.meta == e["meta_all"])
    assert list(p.bq[0, :16]) == e["bq_block0"]
    assert list(p.bq[0, 16:32]) == e["bq_block1"]
    assert np.all(p.bq[0, 32:] == 0)
    assert list(p.bs[0]) == e["bs"]
    assert p.bs[0, 1] != e["bs_block1_other_order"]
    assert list(p.rq[0, :48]) == e["rq_first48"]
    assert np.all(p.rq[0, 48:] == 0)
    assert list(p.rs[0]) == e["rs"]


def _golden_w():
    g = json.load(open(GOLD_W))
    w = np.zeros((64, 2), np.float32)
    for c, col in enumerate(("col0", "col1")):
        for k, v in g["w_nonzero"][col].items():
            w[int(k), c] = v
    return g, w


def _codes_match(wq_row, expect: dict):
    want = np.zeros(wq_row.shape, np.uint8)
    for k, v in expect.items():
        want[int(k)] = v
    return np.array_equal(wq_row, want)


def test_worked_weight_pair_mask():
    """Per-tensor amax (column 1's 0.5, not column 0's 0.25), 32-element blocks, the packed
    payload and both scale views in the tiled layout (hand-worked fixture)."""
    from oracle import layouts as L
    g, w = _golden_w()
    e = g["nvfp4_pair"]
    qw = S.quantize_weight(w, S.NVFP4, S.PAIR48)
    assert np.float32(qw.s_gw).view(np.uint32) == int(e["s_gw_bits"], 16)
    assert qw.ws.tolist() == e["scales"]
    assert _codes_match(qw.wq[0], e["codes_col0"]) and _codes_match(qw.wq[1], e["codes_col1"])
    buf = S.weight_buffers(qw)
    dense, sparse = buf["scales_dense"].reshape(-1), buf["scales_sparse"].reshape(-1)
    assert dense.size == 512 and sparse.size == 512  # one 128 x 4 chunk each
    assert list(dense[0:4]) == e["dense_view_row0"] and list(dense[16:20]) == e["dense_view_row1"]
    assert list(sparse[0:4]) == e["sparse_view_row0"] and list(sparse[16:20]) == e["sparse_view_row1"]
    rest = np.ones(512, bool)
    rest[0:4] = rest[16:20] = False
    assert not dense[rest].any() and not sparse[rest].any()
    codes = buf["codes"].reshape(2, 32)
    assert _codes_match(codes[0], e["packed_col0"]) and _codes_match(codes[1], e["packed_col1"])
    assert L.pack_nibbles(qw.wq).shape == (2, 32)


def test_worked_weight_16_element_blocks():
    """NVFP4 without the pair mask quantises the weight in 16-element blocks: column 1's
    second half-block gets its own scale and its K=20 value a different code."""
    g, w = _golden_w()
    e = g["nvfp4_16"]
    qw = S.quantize_weight(w, S.NVFP4, S.ELEM24)
    assert qw.ws.tolist() == e["scales"]
    assert _codes_match(qw.wq[1], e["codes_col1"])
    assert _codes_match(qw.wq[0], g["nvfp4_pair"]["codes_col0"])


def test_worked_weight_mxfp4():
    g, w = _golden_w()
    e = g["mxfp4"]
    qw = S.quantize_weight(w, S.MXFP4, S.PAIR48)
    assert qw.s_gw == 1.0
    assert qw.ws.tolist() == e["scales"]
    assert _codes_match(qw.wq[0], e["codes_col0"]) and _codes_match(qw.wq[1], e["codes_col1"])


# ----------------------------------------------------------------------------- masks


def _pair_key(g, j):
    a, b = abs(float(g[2 * j])), abs(float(g[2 * j + 1]))
    return (max(a, b), min(a, b))


def test_pair48_brute_force_tiny():
    """For every group, the kept pair set is the C(4,2) subset chosen by exhaustive search:
    the lexicographically largest sorted key list, earliest subset on ties."""
    rng = np.random.default_rng(0)
    # small integers produce many ties
    x = rng.integers(-3, 4, size=(64, 256)).astype(np.float32)
    kept = S.keep_pairs48(x)
    meta = S.canonical_metadata(x, S.PAIR48)
    for m in range(x.shape[0]):
        for gi in range(x.shape[1] // 8):
            grp = x[m, 8 * gi: 8 * gi + 8]
            best = None
            for sub in itertools.combinations(range(4), 2):
                keys = sorted([_pair_key(grp, j) + (-j,) for j in sub], reverse=True)
                if best is None or keys > best[0]:
                    best = (keys, sub)
            sub = best[1]
            assert tuple(np.nonzero(kept[m, gi])[0]) == sub
            assert meta[m, gi] == sub[0] | (sub[1] << 2)


def test_elem24_brute_force_tiny():
    rng = np.random.default_rng(1)
    x = rng.integers(-2, 3, size=(32, 256)).astype(np.float32)
    kept = S.keep_elems24(x)
    meta = S.canonical_metadata(x, S.ELEM24)
    for m in range(x.shape[0]):
        for gi in range(x.shape[1] // 4):
            grp = np.abs(x[m, 4 * gi: 4 * gi + 4])
            best = max(itertools.combinations(range(4), 2),
                       key=lambda s: (sorted([(grp[j], -j) for j in s], reverse=True)))
            assert tuple(np.nonzero(kept[m, gi])[0]) == best
            assert meta[m, gi] == best[0] | (best[1] << 2)


@pytest.mark.parametrize("mask", [S.PAIR48, S.ELEM24])
def test_mask_invariants(mask):
    rng = np.random.default_rng(2)
    x = heavy_activations(rng, 32, 1024).values
    keep = S.keep_mask(x, mask)
    gs = 8 if mask == S.PAIR48 else 4
    k = keep.reshape(32, -1, gs)
    assert np.all(k.sum(-1) == gs // 2)  # exactly N of M survive per group
    a = np.abs(x).reshape(32, -1, gs)
    # the largest |x| of every group always survives (the outlier is captured)
    top = np.argmax(a, axis=-1)
    assert np.all(np.take_along_axis(k, top[..., None], -1))
    if mask == S.ELEM24:
        kept_min = np.where(k, a, np.inf).min(-1)
        drop_max = np.where(~k, a, -np.inf).max(-1)
        assert np.all(kept_min >= drop_max)


# ----------------------------------------------------------------------------- quantisation


def _nearest_value_check(x, codes, d):
    """Every code is the nearest E2M1 grid point of x/d (brute force over the 8 magnitudes,
    saturating at 6)."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    t = np.minimum(np.abs(x.astype(np.float64) / d), 6.0)
    got = np.abs(F.e2m1_decode(codes))
    best = np.abs(t[..., None] - grid).min(-1)
    assert np.all(np.abs(t - got) == best)


@pytest.mark.parametrize("fmt", [S.NVFP4, S.MXFP4])
@pytest.mark.parametrize("mask", [S.PAIR48, S.ELEM24])
def test_backbone_plus_residual_is_exact(fmt, mask):
    """deq(Q(backbone)) + r == x bit-exactly before the residual is quantised."""
    rng = np.random.default_rng(3)
    x = heavy_activations(rng, 64, 2048).values
    p = S.prepare(x, fmt, mask)
    assert np.array_equal((p.b_deq + p.r).astype(np.float32), x)
    assert np.array_equal(p.b_deq.astype(np.float64) + p.r.astype(np.float64), x.astype(np.float64))


def test_nvfp4_scale_and_codes_are_nearest():
    rng = np.random.default_rng(4)
    x = heavy_activations(rng, 16, 1024).values
    s_g, k = S.tensor_scales(np.abs(x).max())
    v = x.reshape(16, -1, 16)
    codes, sf, deq = S.quant_blocks_nv(v, s_g, k)
    a = np.abs(v).max(-1)
    # the scale argument is formed in float32 (the precision the recipe fixes)
    t = (a * k).astype(np.float32).astype(np.float64)
    # k is 1 / (6 s_g) up to the two float32 roundings
    assert abs(float(k) * 6 * float(s_g) - 1) < 2.5e-7
    # sf is the nearest E4M3 value to t (saturating at 448), by brute force over the table
    best = np.abs(np.minimum(t, 448)[..., None] - F.E4M3_TABLE).min(-1)
    assert np.array_equal(np.abs(np.minimum(t, 448) - F.e4m3_decode(sf)), best)
    d = (F.e4m3_decode(sf).astype(np.float32) * s_g).astype(np.float32)
    inv = (np.float32(1) / d).astype(np.float32)
    # codes: nearest grid point of the float32 product x * (1/d)
    _nearest_value_check((v * inv[..., None]).astype(np.float32), codes, 1.0)
    # the block's largest element lands on the top code (6) for normal-range scales
    amax_pos = np.argmax(np.abs(v), -1)
    top = np.take_along_axis(codes, amax_pos[..., None], -1)[..., 0] & 7
    normal = F.e4m3_decode(sf) >= 2.0 ** -6
    assert np.all(top[normal] == 7)


def test_mxfp4_scale_is_floor_log2_minus_2():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((200, 32)) * 2.0 ** rng.integers(-20, 20, (200, 1))).astype(np.float32)
    codes, e8, deq = S.quant_blocks_mx(v)
    a = np.abs(v).max(-1)
    # 2^(e+2) <= amax < 2^(e+3): the amax maps into [4, 8) before rounding
    e = e8.astype(np.int64) - 127
    assert np.all((2.0 ** (e + 2) <= a) & (a < 2.0 ** (e + 3)))
    _nearest_value_check(v, codes, (2.0 ** e)[:, None])


def test_zero_tensor_gives_zero_codes():
    x = np.zeros((4, 256), np.float32)
    for fmt in (S.NVFP4, S.MXFP4):
        p = S.prepare(x, fmt, S.PAIR48)
        assert np.all(p.bq == 0) and np.all(p.rq == 0)
        if fmt == S.NVFP4:
            assert p.s_g == 0 and np.all(p.bs == 0) and np.all(p.rs == 0)
        else:
            assert np.all(p.bs == 0)


@pytest.mark.parametrize("fmt", [S.NVFP4, S.MXFP4])
def test_residual_recovers_error_on_outlier_inputs(fmt):
    """Reconstruction error of SharQ <= plain FP4 of X, and <= the ablation that forms the
    residual against the unquantised backbone (the referee's "what would settle it")."""
    rng = np.random.default_rng(6)
    x = heavy_activations(rng, 128, 4096).values
    p = S.prepare(x, fmt, S.PAIR48)
    err = np.linalg.norm(p.b_deq + p.r_deq - x)
    _, _, plain = S.quant_blocks(fmt, x.reshape(128, -1, S.residual_block(fmt)),
                                 S.tensor_scales(np.abs(x).max()))
    err_plain = np.linalg.norm(plain.reshape(x.shape) - x)
    pu = S.prepare(x, fmt, S.PAIR48, residual_ref="unquantized")
    err_unq = np.linalg.norm(pu.b_deq + pu.r_deq - x)
    assert err < 0.5 * err_plain
    assert err < err_unq


def test_weight_views_agree():
    rng = np.random.default_rng(7)
    w = rng.normal(0, 0.02, (512, 256)).astype(np.float32)
    qw = S.quantize_weight(w, S.NVFP4, S.PAIR48)
    dense = S.weight_scale_view(qw, 16)
    sparse = S.weight_scale_view(qw, 32)
    assert np.array_equal(dense[:, 0::2], sparse) and np.array_equal(dense[:, 1::2], sparse)
