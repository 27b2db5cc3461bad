"""Pins of the oracle's ablation modes (the page's referee asks for a residual against the
unquantised sparse values, a static instead of an input-adaptive mask, and direct FP4
without the decomposition): closed forms, equivalences between independent code paths,
and the direction of the reconstruction errors on outlier-heavy inputs."""
import numpy as np
import pytest

from oracle import sharq as S
from workloads import heavy_activations

F32 = np.float32


def _x(M=64, K=512, seed=0, per_row=True):
    return heavy_activations(np.random.default_rng(seed), M, K, per_row=per_row).values


def _recon(p):
    """float64 reconstruction deq(backbone) + deq(residual) in the tensor's units."""
    out = S.backbone_values(p) * float(p.s_g if p.fmt == S.NVFP4 else 1.0)
    if p.residual:
        out = out + p.r_deq.astype(np.float64)
    return out


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_given_mask_equal_to_adaptive_reproduces_the_method(fmt):
    x = _x()
    a = S.act_buffers(S.prepare(x, fmt, S.PAIR48))
    b = S.act_buffers(S.prepare(x, fmt, S.PAIR48_GIVEN, given=S.keep_pairs48(x)))
    assert a.keys() == b.keys()
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_static_mask_equals_adaptive_when_rows_repeat():
    row = _x(1, 512, seed=3)
    x = np.repeat(row, 8, axis=0)
    assert np.array_equal(S.static_keep_pairs48(x, 8), S.keep_pairs48(x))


def test_static_mask_keeps_two_pairs_everywhere_and_the_same_in_every_row():
    x = _x(32, 1024, seed=4)
    g = S.static_keep_pairs48(x, 32)
    assert np.all(g.sum(axis=-1) == 2)
    assert np.all(g == g[:1])


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_unquantized_reference_residual_is_the_masked_out_part(fmt):
    """r = x - backbone: exactly 0 where the mask keeps, exactly x elsewhere."""
    x = _x(seed=5)
    p = S.prepare(x, fmt, S.PAIR48, residual_ref="unquantized")
    assert np.all(p.r[p.keep] == 0)
    assert np.array_equal(p.r[~p.keep], x[~p.keep])


def test_no_mask_equals_element_mask_when_groups_hold_two_nonzeros():
    """With at most two non-zeros in every 4-group, the 2:4 backbone is all of x, so its
    FP4 values equal plain FP4 of x (independent paths: the 2:4 selection vs keep-all)."""
    rng = np.random.default_rng(6)
    x = _x(32, 512, seed=6)
    z = np.zeros_like(x).reshape(32, -1, 4)
    for g in range(z.shape[1]):
        cols = rng.choice(4, 2, replace=False)
        z[:, g, cols] = 1
    x = (x * z.reshape(x.shape)).astype(F32)
    for fmt in ("nvfp4", "mxfp4"):
        a = S.prepare(x, fmt, S.NONE, residual=False)
        b = S.prepare(x, fmt, S.ELEM24, residual=False)
        assert np.array_equal(S.backbone_values(a), S.backbone_values(b))
        assert np.array_equal(a.bs, b.bs)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_ablation_error_ordering_on_outlier_heavy_inputs(fmt):
    """Reconstruction error (Frobenius): the method <= each ablation on per-row outliers;
    plain FP4 with a dense FP4 residual (two dense terms) <= plain FP4 alone."""
    x = _x(256, 1024, seed=7, per_row=True)
    err = lambda p: np.linalg.norm(x - _recon(p))
    method = err(S.prepare(x, fmt, S.PAIR48))
    unq = err(S.prepare(x, fmt, S.PAIR48, residual_ref="unquantized"))
    static = err(S.prepare(x, fmt, S.PAIR48_GIVEN, given=S.static_keep_pairs48(x, 256)))
    plain = err(S.prepare(x, fmt, S.NONE, residual=False))
    plain2 = err(S.prepare(x, fmt, S.NONE, residual=True))
    assert method <= unq
    assert method <= static
    assert method <= plain
    assert plain2 <= plain


def test_own_residual_scale_is_plain_nvfp4_of_the_residual():
    """The variant with the residual's own tensor scale quantises r exactly as plain NVFP4
    (no mask, no residual) quantises the tensor r: two independent paths."""
    x = _x(64, 1024, seed=8)
    p = S.prepare(x, S.NVFP4, S.PAIR48, residual_scale="own")
    q = S.prepare(p.r, S.NVFP4, S.NONE, residual=False)
    assert np.array_equal(p.rq, q.bq) and np.array_equal(p.rs, q.bs)
    assert p.s_r == q.s_g
    assert p.s_r < p.s_g  # amax|r| < amax|x| on outlier-heavy rows


def test_own_residual_scale_changes_little_on_outlier_heavy_inputs():
    """Both variants approximate the same product; on these inputs the E4M3 block scales
    already carry the residual's range, so the two results are close."""
    from workloads import gaussian_weight
    x = _x(64, 1024, seed=9)
    w = gaussian_weight(np.random.default_rng(10), 1024, 256).values
    qw = S.quantize_weight(w)
    y_shared = S.linear(S.prepare(x), qw)
    y_own = S.linear(S.prepare(x, residual_scale="own"), qw)
    exact = x.astype(np.float64) @ w.astype(np.float64)
    e = lambda y: np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert abs(e(y_own) - e(y_shared)) < 0.1 * e(y_shared)


def test_two_accumulator_product_is_sparse_part_plus_plain_nvfp4_of_the_residual():
    """The own-scale variant's Y: its backbone part is the sparse-only product, and its
    residual part is the product of plain NVFP4 of r (no mask, own tensor scale) with the
    weight's dense view; both computed by other code paths (the sparse-only product and
    the no-mask preparation), so a wrong scale or a dropped term fails here."""
    from workloads import gaussian_weight
    x = _x(48, 512, seed=11)
    w = gaussian_weight(np.random.default_rng(12), 512, 128).values
    p = S.prepare(x, S.NVFP4, S.PAIR48, residual_scale="own")
    qw = S.quantize_weight(w, S.NVFP4, S.PAIR48)  # one code payload for both paths
    y = S.linear(p, qw)
    sparse = S.linear_sparse_only(p, qw)
    plain_r = S.linear(S.prepare(p.r, S.NVFP4, S.NONE, residual=False), qw)
    np.testing.assert_allclose(y, sparse + plain_r, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_weight_block_study_orders_the_errors():
    """The 32-element weight block that lets one FP4 payload serve both scale views costs
    weight accuracy against 16-element NVFP4 blocks: its weight error is larger (each scale
    covers twice the values), and the Y error follows; both sit above the activations'
    own share (activations quantised, weight exact)."""
    from oracle import weight_block_study as WB
    from workloads import gaussian_weight
    rng = np.random.default_rng(5)
    x = heavy_activations(rng, 32, 1024).values
    w = gaussian_weight(rng, 1024, 512).values
    r = WB.study(x, w)
    assert r["16"]["w_err"] < r["32"]["w_err"] < 0.2
    assert r["16"]["y_err"] < r["32"]["y_err"]
    assert r["act_only_y_err"] < r["16"]["y_err"]
