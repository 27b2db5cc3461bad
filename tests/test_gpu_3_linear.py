"""GPU parity of the fused sparse + dense FP4 GEMM against the oracle's float64 product of
the same dequantised operands.

Tolerances: the oracle forms Y64 = s_g * s_gw * sum_k (B + R)[m,k] * W[n,k] exactly (every
operand is a short dyadic number) with float64 sums. The kernel accumulates the same
products in FP32 tensor memory, so for K <= 16384 its relative error is a few 1e-7; the
float32 output is held to 1e-5 relative Frobenius error. The bf16 output is compared with
bf16(Y64) rounded once from float64: the two differ only where the FP32 accumulation
moves a value across a bf16 rounding boundary, which the 1e-3 bound (the target's) covers
with wide margin."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import sharq as S
from tests.gpu_helpers import cfg_of, rel_fro, to_device, upload_act, upload_weight
from workloads import BF16, F16, gaussian_weight, heavy_activations, tiny_activations

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 1e-3


def gpu_linear(act, w, out_f32=False):
    import fp4_sparse_dense_b200 as sq
    import torch
    y = sq.linear(act, w, out_dtype=torch.float32 if out_f32 else torch.bfloat16)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    return y.float().cpu().numpy().astype(np.float64)


def check_y(y_gpu, y64, bf16_out):
    if bf16_out:
        err = rel_fro(y_gpu, F.bf16_round(y64))
        assert err <= TOL_BF16, err
    else:
        err = rel_fro(y_gpu, y64)
        assert err <= TOL_F32, err
    return err


GEMM_CASES = [
    # fmt, mask, residual, M, K, N
    ("nvfp4", "pair48", True, 128, 256, 256),
    ("nvfp4", "pair48", True, 1, 512, 128),
    ("nvfp4", "pair48", True, 100, 1024, 384),
    ("nvfp4", "pair48", True, 257, 768, 512),
    ("nvfp4", "pair48", False, 200, 512, 256),
    ("nvfp4", "elem24", True, 130, 512, 256),
    ("nvfp4", "elem24", False, 64, 256, 128),
]
PAIR_CASES = [  # M >= 256 and N % 256 == 0: the CTA-pair kernel (odd 128-row counts included)
    ("nvfp4", "pair48", True, 256, 512, 256),
    ("nvfp4", "pair48", True, 300, 1024, 512),
    ("nvfp4", "pair48", True, 640, 768, 768),
    ("nvfp4", "pair48", False, 512, 256, 256),
    ("nvfp4", "elem24", True, 384, 512, 256),
    ("mxfp4", "pair48", True, 513, 512, 256),
    ("mxfp4", "elem24", True, 256, 256, 512),
    # 80 pair tiles for 74 CTA pairs: some pairs run a second tile (K / 256 even, so the
    # next tile's scales are copied while the epilogue drains the accumulator)
    ("nvfp4", "pair48", True, 2048, 512, 2560),
    ("nvfp4", "pair48", False, 2048, 512, 2560),
    ("mxfp4", "pair48", True, 2048, 512, 2560),
    ("nvfp4", "elem24", True, 2048, 512, 2560),
]
MX_CASES = [
    ("mxfp4", "pair48", True, 128, 512, 256),
    ("mxfp4", "pair48", True, 77, 1024, 128),
    ("mxfp4", "elem24", True, 150, 512, 256),
    ("mxfp4", "pair48", False, 64, 256, 128),
]


@pytest.mark.parametrize("fmt,mask,residual,M,K,N", GEMM_CASES + MX_CASES + PAIR_CASES)
@pytest.mark.parametrize("out_f32", [True, False])
def test_gemm_on_oracle_operands(fmt, mask, residual, M, K, N, out_f32):
    """The GEMM alone: operands are the oracle's bytes uploaded to the GPU."""
    rng = np.random.default_rng(M + K + N)
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    p = S.prepare(x.values, fmt, mask, residual=residual)
    qw = S.quantize_weight(w.values, fmt, mask)
    cfg = cfg_of(fmt, mask, residual)
    act = upload_act(S.act_buffers(p), M, K, cfg)
    wt = upload_weight(S.weight_buffers(qw), K, N, cfg)
    check_y(gpu_linear(act, wt, out_f32), S.linear(p, qw), not out_f32)


@pytest.mark.parametrize("fmt,mask,residual,M,K,N", GEMM_CASES + MX_CASES + PAIR_CASES)
def test_end_to_end(fmt, mask, residual, M, K, N):
    """prepare + quantize_weight + linear on the GPU vs the oracle chain."""
    import fp4_sparse_dense_b200 as sq
    rng = np.random.default_rng(3 * M + K + N)
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of(fmt, mask, residual)
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    p = S.prepare(x.values, fmt, mask, residual=residual)
    qw = S.quantize_weight(w.values, fmt, mask)
    check_y(gpu_linear(act, wt, True), S.linear(p, qw), False)


def test_residual_off_is_sparse_only_product():
    import fp4_sparse_dense_b200 as sq
    rng = np.random.default_rng(9)
    M, K, N = 96, 512, 256
    x = heavy_activations(rng, M, K)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of("nvfp4", "pair48", False)
    y = gpu_linear(sq.prepare(to_device(x), cfg), sq.quantize_weight(to_device(w), cfg), True)
    p = S.prepare(x.values)
    qw = S.quantize_weight(w.values)
    assert rel_fro(y, S.linear_sparse_only(p, qw)) <= TOL_F32


def test_tiny_config_end_to_end():
    """X[16x256] fp16 with 4 outlier channels, W[256x128] fp16, element 2:4, NVFP4."""
    import fp4_sparse_dense_b200 as sq
    x = tiny_activations()
    w = gaussian_weight(np.random.default_rng(1), 256, 128, F16)
    cfg = cfg_of("nvfp4", "elem24")
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    p = S.prepare(x.values, "nvfp4", "elem24")
    qw = S.quantize_weight(w.values, "nvfp4", "elem24")
    y64 = S.linear(p, qw)
    check_y(gpu_linear(act, wt, True), y64, False)
    check_y(gpu_linear(act, wt, False), y64, True)


@pytest.mark.parametrize("name,M,K,N,per_row", [
    ("attn_proj", 2048, 4096, 4096, False),
    ("mlp_gate_up", 4096, 4096, 14336, False),
    ("mlp_down_decode", 1, 14336, 4096, True),
    ("mlp_down_decode", 64, 14336, 4096, True),
    ("mlp_down_prefill", 4096, 14336, 4096, True),
])
def test_full_size_sampled_outputs(name, M, K, N, per_row):
    """Benchmark shapes in the benchmark's launch configuration (bf16 output): sampled
    rows x sampled columns of Y against the oracle on those rows and columns."""
    import fp4_sparse_dense_b200 as sq
    rng = np.random.default_rng(M + N)
    x = heavy_activations(rng, M, K, per_row=per_row)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of("nvfp4", "pair48")
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    y = gpu_linear(act, wt, False)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(M, 30), replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 200, replace=False)]))
    p = S.prepare(x.values[rows], amax=S.amax_of(x.values))
    qw = S.quantize_weight(w.values[:, cols], amax=S.amax_of(w.values))
    y64 = S.linear(p, qw)
    check_y(y[np.ix_(rows, cols)], y64, True)


@pytest.mark.parametrize("M,K,N", [(1, 14336, 4096), (8, 14336, 4096), (16, 14336, 4096),
                                   (16, 4096, 1024),
                                   (64, 14336, 4096), (100, 2048, 384),
                                   # 16, 17 and 28 K ranges: the summing kernel loads the
                                   # partials of up to 16 splits per batch
                                   (2, 8192, 256), (3, 8704, 256), (1, 14336, 128)])
def test_split_k_decode(M, K, N):
    """Decode-sized M: the split-K path (caller workspace, fixed-order reduction) agrees with
    the oracle and with the unsplit path, and repeats bit-identically."""
    import fp4_sparse_dense_b200 as sq
    import torch
    rng = np.random.default_rng(M * 31 + N)
    x = heavy_activations(rng, M, K, per_row=True)
    w = gaussian_weight(rng, K, N)
    cfg = cfg_of("nvfp4", "pair48")
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    ws = sq.linear_workspace(M, N, K, cfg)
    assert ws is not None and ws.numel() >= M * N * 4 * 2
    y_split = sq.linear(act, wt, out_dtype=torch.float32, workspace=ws)
    y_split2 = sq.linear(act, wt, out_dtype=torch.float32, workspace=ws)
    y_plain = sq.linear(act, wt, out_dtype=torch.float32, workspace=None)
    y_bf16 = sq.linear(act, wt, workspace=ws)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    assert torch.equal(y_split, y_split2)
    p = S.prepare(x.values)
    qw = S.quantize_weight(w.values)
    y64 = S.linear(p, qw)
    check_y(y_split.cpu().numpy().astype(np.float64), y64, False)
    check_y(y_plain.cpu().numpy().astype(np.float64), y64, False)
    check_y(y_bf16.float().cpu().numpy().astype(np.float64), y64, True)


@pytest.mark.parametrize("out_f32", [True, False])
def test_split_k_rows_independent_of_other_rows(out_f32):
    """Split-K rows do not depend on the other rows of the call: rows 0..7 of a 16-row input
    whose rows 8..15 are rows 0..7 halved (same tensor amax, so the same codes and scales
    for rows 0..7, and the same K ranges, since both shapes have one row block) give Y
    bit-identical to an 8-row call, the partials being summed in the same fixed order."""
    import fp4_sparse_dense_b200 as sq
    import torch
    K, N = 14336, 4096
    rng = np.random.default_rng(808)
    x8 = to_device(heavy_activations(rng, 8, K, per_row=True))
    x16 = torch.cat([x8, x8 * 0.5])
    wt = sq.quantize_weight(to_device(gaussian_weight(rng, K, N)), cfg_of("nvfp4", "pair48"))
    cfg = cfg_of("nvfp4", "pair48")
    dt = torch.float32 if out_f32 else torch.bfloat16
    y8 = sq.linear(sq.prepare(x8, cfg), wt, out_dtype=dt, workspace=sq.linear_workspace(8, N, K, cfg))
    y16 = sq.linear(sq.prepare(x16, cfg), wt, out_dtype=dt,
                    workspace=sq.linear_workspace(16, N, K, cfg))
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    assert torch.equal(y8, y16[:8])


def test_split_k_workspace_reused_across_shapes():
    """One workspace, sized for the largest shape, serves several decode shapes in turn; each
    call's result is independent of what earlier calls left in it."""
    import fp4_sparse_dense_b200 as sq
    import torch
    K, N = 14336, 4096
    cfg = cfg_of("nvfp4", "pair48")
    rng = np.random.default_rng(123)
    w = gaussian_weight(rng, K, N)
    wt = sq.quantize_weight(to_device(w), cfg)
    qw = S.quantize_weight(w.values)
    ws = sq.linear_workspace(64, N, K, cfg)
    for M in (64, 1, 16, 64, 8):
        x = heavy_activations(rng, M, K, per_row=True)
        act = sq.prepare(to_device(x), cfg)
        assert sq.linear_workspace(M, N, K, cfg).numel() <= ws.numel()
        y = sq.linear(act, wt, out_dtype=torch.float32, workspace=ws).cpu().numpy()
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
        y64 = S.linear(S.prepare(x.values), qw)
        assert rel_fro(y, y64) <= 1e-5, M



@pytest.mark.parametrize("M", [1, 16])
def test_weight_requantised_just_before_linear(M):
    """At decode-sized M the GEMM may load its weight while the kernel launched just before
    it still runs, but only when that kernel is a preparation's or a linear call's. A weight
    re-quantised into the same buffers right before sharq_linear must be read in full: the
    result equals that of the new weight quantised before the preparation, bit for bit, and
    differs from the old weight's."""
    import fp4_sparse_dense_b200 as sq
    import torch
    K, N = 14336, 4096
    cfg = cfg_of("nvfp4", "pair48")
    rng = np.random.default_rng(4242 + M)
    x = to_device(heavy_activations(rng, M, K, per_row=True))
    w_old = to_device(gaussian_weight(rng, K, N))
    w_new = to_device(gaussian_weight(rng, K, N))
    ws = sq.linear_workspace(M, N, K, cfg)
    dt = torch.float32
    wt = sq.quantize_weight(w_old, cfg)
    act = sq.prepare(x, cfg)
    y_old = sq.linear(act, wt, out_dtype=dt, workspace=ws)       # after a preparation
    sq.quantize_weight(w_new, cfg, out=wt)                       # same buffers, new weight
    y_late = sq.linear(act, wt, out_dtype=dt, workspace=ws)      # right after the quantisation
    wt2 = sq.quantize_weight(w_new, cfg)
    y_ref = sq.linear(sq.prepare(x, cfg), wt2, out_dtype=dt, workspace=ws)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    assert torch.equal(y_late, y_ref)
    assert not torch.equal(y_old, y_ref)
