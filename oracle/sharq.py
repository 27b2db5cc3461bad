"""CPU oracle of the SharQ sparse-dense FP4 linear layer.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / reference leg of bench.py, never by the product path. It shares no
code with the CUDA kernels.

What it computes follows the SharQ page ("SharQ: Bridging Activation Sparsity and FP4
Quantization for LLM Inference", pith.science 2606.26587), sections "The pith",
"Core claim" and the arXiv abstract:

1. per activation tensor, an input-adaptive N:M mask along K extracts an
   outlier-dominated sparse backbone (largest |x| kept);
2. the backbone is quantised to FP4 (NVFP4: E2M1 codes, E4M3 scale per block, FP32
   tensor scale; MXFP4: E8M0 scale per block);
3. a dense residual is defined against the *quantised* backbone, r = x - deq(Q(b)),
   and quantised to FP4 with its own block scales;
4. Y = sparse-FP4-GEMM(backbone, W) + dense-FP4-GEMM(r, W), both over one FP4 weight
   payload whose scales are presented in a path-specific view.

The pages give no equations. Where they are silent the oracle takes these readings
(listed with their reasons in the design notes):

* mask ``pair48``: in every group of 8 consecutive K elements keep 2 of the 4 adjacent
  pairs; pairs ranked by (max |x| of the pair, then min |x| of the pair), ties to the
  lower pair index. This is the pattern the sm_100a sparse FP4 MMA accepts.
* mask ``elem24``: in every group of 4 keep the 2 largest |x|, ties to the lower index.
* NVFP4 tensor constants from amax|X|, each one float32 division: the tensor scale
  s_g = amax / (6*448) and the block-scale factor k = 448 / amax (= 1 / (6 s_g) in exact
  arithmetic); block scale sf = E4M3_rne_satfinite(a * k) with a the block's max |x|;
  d = E4M3(sf) * s_g; inv = 1 / d (one correctly rounded reciprocal per block);
  code = E2M1_rne(x * inv) (code 0 when d == 0).
  Dequantised value deq = (E2M1(q) * E4M3(sf)) * s_g, all in float32 with one rounding
  per operation.
* MXFP4 (OCP MX): e = clamp(floor(log2 a) - 2, -127, 127), scale 2^e as E8M0 code
  e+127, code = E2M1_rne(x * 2^-e); a == 0 gives code 0 for scale and elements.
* Block domains (forced by the MMA that consumes each operand): the residual uses
  16-element (NVFP4) / 32-element (MXFP4) blocks along K. The backbone uses 32
  logical K positions per scale for ``pair48`` (= 16 kept values, the granularity of
  the sparse block-scaled MMA), and the residual's block size for ``elem24`` (where the
  backbone is stored zero-filled and runs through the dense MMA). The weight uses
  32-element blocks when ``pair48`` is on, so that one set of codes is valid under both
  the 16-granular view (dense MMA) and the 32-granular view (sparse MMA).
* the residual reuses the activation tensor scale s_g, so both GEMMs share one
  accumulator and one epilogue factor alpha = s_g * s_gw.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import formats as F

NVFP4 = "nvfp4"
MXFP4 = "mxfp4"
PAIR48 = "pair48"
ELEM24 = "elem24"
# ablation modes (the page's referee asks for them; see prepare): the pair-wise 4:8 mask
# supplied by the caller (e.g. a static, per-tensor channel set) and no mask (plain FP4)
PAIR48_GIVEN = "pair48_given"
NONE = "none"


def is_pair(mask: str) -> bool:
    """Masks whose backbone is stored compressed and runs through the sparse MMA."""
    return mask in (PAIR48, PAIR48_GIVEN)

F32 = np.float32
GLOBAL_DIV = F32(6.0 * 448.0)  # E2M1 max * E4M3 max


# ----------------------------------------------------------------------------- blocks


def residual_block(fmt: str) -> int:
    return 16 if fmt == NVFP4 else 32


def backbone_block(fmt: str, mask: str) -> int:
    """Logical K positions covered by one backbone scale."""
    if is_pair(mask):
        return 32
    return residual_block(fmt)


def weight_block(fmt: str, mask: str) -> int:
    if fmt == MXFP4:
        return 32
    return 32 if is_pair(mask) else 16


def dense_view_block(fmt: str) -> int:
    """Scale granularity along K of the dense block-scaled MMA (NVFP4 4X / MXFP4 2X)."""
    return 16 if fmt == NVFP4 else 32


SPARSE_VIEW_BLOCK = 32  # sparse block-scaled MMA: 4 scales per 128 logical K


# ----------------------------------------------------------------------------- scales


def amax_of(x: np.ndarray) -> np.float32:
    return F32(np.max(np.abs(x.astype(F32)))) if x.size else F32(0)


def tensor_scales(amax: np.float32) -> tuple[np.float32, np.float32]:
    """NVFP4 per-tensor constants from amax|X| (float32, one division each):
    s_g = amax / 2688 (the FP32 tensor scale, used to dequantise) and
    k = 448 / amax (the block-scale factor: a / 6 / s_g in exact arithmetic)."""
    amax = F32(amax)
    s_g = F32(amax / GLOBAL_DIV)
    with np.errstate(divide="ignore"):
        k = F32(F32(448.0) / amax) if amax > 0 else F32(np.inf)
    return s_g, k


def tensor_scale(x: np.ndarray) -> np.float32:
    """NVFP4 FP32 tensor scale s_g = amax|X| / 2688."""
    return tensor_scales(amax_of(x))[0]


def quant_blocks_nv(v: np.ndarray, s_g: np.float32, k: np.float32):
    """NVFP4 quantisation of blocks along the last axis.

    v: float32 [..., nblk, B]; s_g, k from tensor_scales(). Returns (codes uint8
    [..., nblk, B], sf uint8 [..., nblk], deq float32 [..., nblk, B]) with
    sf = E4M3(a * k), deq = (E2M1(q) * E4M3(sf)) * s_g in float32.
    """
    v = v.astype(F32)
    a = np.max(np.abs(v), axis=-1)  # float32, exact
    if s_g == 0:
        sf = np.zeros(a.shape, np.uint8)
        codes = np.zeros(v.shape, np.uint8)
        return codes, sf, np.zeros(v.shape, F32)
    t = (a * F32(k)).astype(F32)  # one float32 product per block
    sf = F.e4m3_encode_unsigned(t.astype(F32))
    sf_val = F.e4m3_decode(sf).astype(F32)  # exact
    d = (sf_val * s_g).astype(F32)
    # one correctly rounded reciprocal per block, then one float32 product per element
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (F32(1.0) / d).astype(F32)
        ratio = (v * inv[..., None]).astype(F32)
    codes = np.where(d[..., None] > 0, F.e2m1_encode(np.where(d[..., None] > 0, ratio, 0)), 0)
    codes = codes.astype(np.uint8)
    q_val = F.e2m1_decode(codes).astype(F32)
    deq = ((q_val * sf_val[..., None]).astype(F32) * s_g).astype(F32)
    return codes, sf, deq


def quant_blocks_mx(v: np.ndarray):
    """MXFP4 (OCP MX) quantisation of blocks along the last axis.

    Returns (codes uint8, e8m0 code uint8, deq float32); deq = E2M1(q) * 2^e exactly.
    """
    v = v.astype(F32)
    a = np.max(np.abs(v), axis=-1).astype(np.float64)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = m * 2^ex, m in [0.5, 1)
    e = np.clip(ex - 1 - 2, -127, 127)  # floor(log2 a) - emax(E2M1)
    e = np.where(a > 0, e, -127)
    scale = np.ldexp(1.0, -e).astype(F32)  # 2^-e, exact in float32 for e in [-127, 127]
    x_scaled = (v * scale[..., None]).astype(F32)
    codes = F.e2m1_encode(x_scaled)
    codes = np.where(a[..., None] > 0, codes, 0).astype(np.uint8)
    deq = (F.e2m1_decode(codes) * np.ldexp(1.0, e)[..., None]).astype(F32)
    return codes, (e + 127).astype(np.uint8), deq


def quant_blocks(fmt: str, v: np.ndarray, scales: tuple):
    """scales = tensor_scales(amax) for NVFP4 (ignored for MXFP4)."""
    if fmt == NVFP4:
        return quant_blocks_nv(v, *scales)
    return quant_blocks_mx(v)


def scale_value(fmt: str, sf: np.ndarray) -> np.ndarray:
    """Block-scale codes -> float64 values (without the tensor scale)."""
    return F.e4m3_decode(sf) if fmt == NVFP4 else F.e8m0_decode(sf)


# ----------------------------------------------------------------------------- masks


def _top2_of_4(hi: np.ndarray, lo: np.ndarray) -> np.ndarray:
    """Boolean [..., 4]: the 2 of 4 candidates with the largest key (hi, then lo), ties
    to the lower candidate index. A candidate is kept when fewer than 2 others beat it."""
    n_beaten_by = np.zeros(hi.shape, np.int64)
    for j in range(4):
        for i in range(4):
            if i == j:
                continue
            beats = (hi[..., i] > hi[..., j]) | (
                (hi[..., i] == hi[..., j]) & ((lo[..., i] > lo[..., j])
                                              | ((lo[..., i] == lo[..., j]) & (i < j))))
            n_beaten_by[..., j] += beats
    return n_beaten_by < 2


def keep_pairs48(x: np.ndarray) -> np.ndarray:
    """Boolean [M, K/8, 4]: kept pairs of every 8-group (pair j = elements 2j, 2j+1).

    Pairs are ranked by the larger |x| of the pair, then by the smaller |x|, then by
    the lower pair index; the top 2 are kept.
    """
    M, K = x.shape
    a = np.abs(x.astype(F32)).reshape(M, K // 8, 4, 2)
    return _top2_of_4(a.max(axis=-1), a.min(axis=-1))


def keep_elems24(x: np.ndarray) -> np.ndarray:
    """Boolean [M, K/4, 4]: the 2 largest |x| of every 4-group (ties to the lower index)."""
    M, K = x.shape
    a = np.abs(x.astype(F32)).reshape(M, K // 4, 4)
    return _top2_of_4(a, np.zeros_like(a))


def static_keep_pairs48(x_stat: np.ndarray, M: int) -> np.ndarray:
    """Static pair-wise 4:8 mask (ablation: the channel set fixed per tensor instead of
    chosen per row): the pairs are ranked as in keep_pairs48, but on the per-column max |x|
    of the statistics tensor x_stat, and the same kept pairs serve all M rows.
    Boolean [M, K/8, 4]."""
    col = np.max(np.abs(np.asarray(x_stat, F32)), axis=0, keepdims=True)  # [1, K]
    return np.broadcast_to(keep_pairs48(col), (M,) + keep_pairs48(col).shape[1:]).copy()


def keep_mask(x: np.ndarray, mask: str, given=None) -> np.ndarray:
    """Boolean [M, K]: True where the backbone keeps the element. `given` is the kept pairs
    ([M, K/8, 4]) of the pair48_given mode."""
    M, K = x.shape
    if mask == PAIR48:
        return np.repeat(keep_pairs48(x), 2, axis=-1).reshape(M, K)
    if mask == PAIR48_GIVEN:
        assert given is not None and np.all(np.asarray(given).sum(axis=-1) == 2)
        return np.repeat(np.asarray(given, bool), 2, axis=-1).reshape(M, K)
    if mask == NONE:
        return np.ones((M, K), bool)
    return keep_elems24(x).reshape(M, K)


def canonical_metadata(x: np.ndarray, mask: str, given=None) -> np.ndarray:
    """One nibble per group: i0 | i1 << 2 with i0 < i1 the kept pair indices (pair48)
    or kept element indices (elem24). Shape [M, groups]; empty for the "none" mode."""
    if mask == NONE:
        return np.zeros((x.shape[0], 0), np.uint8)
    if mask == PAIR48:
        kept = keep_pairs48(x)
    elif mask == PAIR48_GIVEN:
        kept = np.asarray(given, bool)
    else:
        kept = keep_elems24(x)
    pos = np.arange(4)
    i0 = np.where(kept, pos, 9).min(axis=-1)
    i1 = np.where(kept, pos, -1).max(axis=-1)
    return (i0 | (i1 << 2)).astype(np.uint8)


# ----------------------------------------------------------------------------- prepare


@dataclass
class Prepared:
    """Canonical (unpacked) result of the activation preparation."""

    fmt: str
    mask: str
    residual: bool
    s_g: np.float32
    keep: np.ndarray  # bool [M, K]
    meta: np.ndarray  # uint8 nibbles [M, groups]
    bq: np.ndarray  # uint8 codes: [M, K/2] compressed (pair48) or [M, K] zero-filled (elem24)
    bs: np.ndarray  # uint8 scale codes [M, K/backbone_block]
    b_deq: np.ndarray  # float32 [M, K]: backbone dequantised at logical positions, 0 elsewhere
    r: np.ndarray | None  # float32 [M, K]: residual before quantisation
    rq: np.ndarray | None  # uint8 codes [M, K]
    rs: np.ndarray | None  # uint8 scale codes [M, K/residual_block]
    r_deq: np.ndarray | None
    s_r: np.float32 | None = None  # the residual's own tensor scale (variant), else None


def prepare(x: np.ndarray, fmt: str = NVFP4, mask: str = PAIR48, residual: bool = True,
            residual_ref: str = "quantized", amax: np.float32 | None = None,
            given=None, residual_scale: str = "shared", amax_r: np.float32 | None = None
            ) -> Prepared:
    """Online sparse-dense decomposition of one activation tensor X[M x K].

    residual_ref="quantized" is the method (r = x - deq(Q(backbone))); "unquantized"
    is the ablation the page's referee asks for (r = x - backbone: zero at kept
    positions). The other referee ablations are masks: "pair48_given" takes the kept
    pairs from `given` (a static mask, e.g. static_keep_pairs48), and "none" keeps every
    element (plain FP4 of x in the residual's block size; with residual on, r = x -
    deq(Q(x)) is a second, dense FP4 term). `amax` overrides the tensor's max |x|, so
    that a sample of rows can be prepared exactly as inside the whole tensor (rows are
    independent once the tensor constants are fixed).

    residual_scale="own" (NVFP4; the variant with two accumulators): the residual gets its
    own tensor scale s_r = amax|r| / 2688 (k_r = 448 / amax|r|) instead of sharing s_g;
    `amax_r` overrides amax|r| for a sample of rows.
    """
    x = np.ascontiguousarray(x, dtype=F32)
    M, K = x.shape
    assert K % 256 == 0
    if fmt == NVFP4:
        sc = tensor_scales(amax_of(x) if amax is None else amax)
    else:
        sc = (F32(1.0), F32(1.0))
    s_g = sc[0]
    keep = keep_mask(x, mask, given)
    meta = canonical_metadata(x, mask, given)
    Bb = backbone_block(fmt, mask)
    if is_pair(mask):
        comp = x[keep].reshape(M, K // 2)  # kept values in K order (row-major boolean gather)
        codes, bs, deq_c = quant_blocks(fmt, comp.reshape(M, -1, 16), sc)
        bq = codes.reshape(M, K // 2)
        b_deq = np.zeros((M, K), F32)
        b_deq[keep] = deq_c.reshape(-1)
    else:
        b = np.where(keep, x, F32(0))
        codes, bs, deq = quant_blocks(fmt, b.reshape(M, -1, Bb), sc)
        bq = codes.reshape(M, K)
        b_deq = np.where(keep, deq.reshape(M, K), F32(0)).astype(F32)
    bs = bs.reshape(M, K // Bb)
    r = rq = rs = r_deq = None
    if residual:
        sub = b_deq if residual_ref == "quantized" else np.where(keep, x, F32(0))
        r = np.where(keep, (x - sub).astype(F32), x).astype(F32)
        Br = residual_block(fmt)
        sc_r = sc
        if residual_scale == "own" and fmt == NVFP4:
            sc_r = tensor_scales(amax_of(r) if amax_r is None else F32(amax_r))
        rc, rsc, rd = quant_blocks(fmt, r.reshape(M, -1, Br), sc_r)
        rq = rc.reshape(M, K)
        rs = rsc.reshape(M, K // Br)
        r_deq = rd.reshape(M, K)
        s_r = sc_r[0] if sc_r is not sc else None
        return Prepared(fmt, mask, residual, s_g, keep, meta, bq, bs, b_deq, r, rq, rs, r_deq,
                        s_r)
    return Prepared(fmt, mask, residual, s_g, keep, meta, bq, bs, b_deq, r, rq, rs, r_deq)


# ----------------------------------------------------------------------------- weight


@dataclass
class QWeight:
    fmt: str
    mask: str
    s_gw: np.float32
    wq: np.ndarray  # uint8 codes [N, K] (K-major, i.e. W transposed)
    ws: np.ndarray  # uint8 scale codes [N, K/weight_block]


def quantize_weight(w: np.ndarray, fmt: str = NVFP4, mask: str = PAIR48,
                    amax: np.float32 | None = None) -> QWeight:
    """W[K x N] -> FP4 codes stored [N x K] (K-major) with block scales along K.

    `amax` overrides max |W| (for quantising a sample of output columns)."""
    wt = np.ascontiguousarray(w.astype(F32).T)  # [N, K]
    N, K = wt.shape
    if fmt == NVFP4:
        sc = tensor_scales(amax_of(wt) if amax is None else amax)
    else:
        sc = (F32(1.0), F32(1.0))
    s_gw = sc[0]
    Bw = weight_block(fmt, mask)
    codes, ws, _ = quant_blocks(fmt, wt.reshape(N, -1, Bw), sc)
    return QWeight(fmt, mask, s_gw, codes.reshape(N, K), ws.reshape(N, K // Bw))


def weight_scale_view(qw: QWeight, granularity: int) -> np.ndarray:
    """The weight's scale codes presented at `granularity` logical K per scale.

    A finer view repeats each code; a coarser view is only valid when the codes agree.
    """
    Bw = weight_block(qw.fmt, qw.mask)
    if granularity == Bw:
        return qw.ws
    if granularity < Bw:
        return np.repeat(qw.ws, Bw // granularity, axis=1)
    raise ValueError("coarser view than the quantisation block")


# ----------------------------------------------------------------------------- values


def backbone_values(p: Prepared) -> np.ndarray:
    """float64 [M, K]: E2M1(q) * block scale at kept positions (tensor scale excluded)."""
    M = p.bq.shape[0]
    K = p.keep.shape[1]
    Bb = backbone_block(p.fmt, p.mask)
    sv = scale_value(p.fmt, p.bs)  # [M, K/Bb]
    out = np.zeros((M, K))
    if is_pair(p.mask):
        vals = F.e2m1_decode(p.bq).reshape(M, K // Bb, 16) * sv[..., None]
        out[p.keep] = vals.reshape(-1)
    else:
        out = (F.e2m1_decode(p.bq).reshape(M, K // Bb, Bb) * sv[..., None]).reshape(M, K)
    return out


def residual_values(p: Prepared) -> np.ndarray:
    M, K = p.rq.shape
    Br = residual_block(p.fmt)
    return (F.e2m1_decode(p.rq).reshape(M, K // Br, Br)
            * scale_value(p.fmt, p.rs)[..., None]).reshape(M, K)


def weight_values(qw: QWeight) -> np.ndarray:
    N, K = qw.wq.shape
    Bw = weight_block(qw.fmt, qw.mask)
    return (F.e2m1_decode(qw.wq).reshape(N, K // Bw, Bw)
            * scale_value(qw.fmt, qw.ws)[..., None]).reshape(N, K)


def alpha(p: Prepared, qw: QWeight) -> float:
    return float(np.float64(p.s_g) * np.float64(qw.s_gw))


def linear(p: Prepared, qw: QWeight, rows: np.ndarray | None = None,
           cols: np.ndarray | None = None) -> np.ndarray:
    """Y = sparse GEMM(backbone, W) + dense GEMM(residual, W), exact operands, float64 sums.

    Y64[m, n] = s_g * s_gw * sum_k (B[m,k] + R[m,k]) * W[n,k]. `rows`/`cols` restrict the
    output to a sample (rows are independent, so sampling is exact).
    """
    A = backbone_values(p)
    Wv = weight_values(qw)
    if cols is not None:
        Wv = Wv[cols]
    if p.residual and p.s_r is not None:
        # two accumulators: each path carries its own tensor scale
        R = residual_values(p)
        if rows is not None:
            A, R = A[rows], R[rows]
        s_gw = float(qw.s_gw) if qw.fmt == NVFP4 else 1.0
        return s_gw * (float(p.s_g) * (A @ Wv.T) + float(p.s_r) * (R @ Wv.T))
    if p.residual:
        A = A + residual_values(p)
    if rows is not None:
        A = A[rows]
    return alpha(p, qw) * (A @ Wv.T)


def linear_sparse_only(p: Prepared, qw: QWeight) -> np.ndarray:
    return alpha(p, qw) * (backbone_values(p) @ weight_values(qw).T)


# ----------------------------------------------------------------------------- device bytes


def act_buffers(p: Prepared) -> dict:
    """The exact bytes the preparation kernel must write, in the HBM layouts of layouts.py."""
    from . import layouts as L
    M, K = p.keep.shape
    out = {"tensor_scale": np.array([p.s_g], F32)}
    out["bq"] = L.pack_nibbles(p.bq).reshape(-1)
    out["bs"] = L.to_scale_layout(p.bs)
    if is_pair(p.mask):
        out["bm"] = L.to_meta48_layout(p.meta)
    elif p.mask == ELEM24:
        out["bm"] = L.to_meta24_layout(p.meta)
    if p.residual:
        out["rq"] = L.pack_nibbles(p.rq).reshape(-1)
        out["rs"] = L.to_scale_layout(p.rs)
    return out


def weight_buffers(qw: QWeight) -> dict:
    """Bytes of the quantised weight: one code payload, two scale views."""
    from . import layouts as L
    out = {"tensor_scale": np.array([qw.s_gw], F32)}
    out["codes"] = L.pack_nibbles(qw.wq).reshape(-1)
    out["scales_dense"] = L.to_scale_layout(weight_scale_view(qw, dense_view_block(qw.fmt)))
    if is_pair(qw.mask):
        out["scales_sparse"] = L.to_scale_layout(weight_scale_view(qw, SPARSE_VIEW_BLOCK))
    return out
