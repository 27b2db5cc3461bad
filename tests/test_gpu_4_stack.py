"""GPU parity on the 8B-shaped layer stack: the seven Llama-3-8B linear shapes (hidden
4096, MLP 14336, GQA kv 1024), NVFP4 and MXFP4, decode to prefill row counts. Sampled rows
and columns of Y (bf16 output) against the oracle on those rows and columns, with the
tensor scales of the whole tensors; the prepared bytes of the sampled rows are bit-exact."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import sharq as S
from tests.gpu_helpers import cfg_of, rel_fro, to_device
from workloads import LLAMA8B_LINEARS, config_problems

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-3


def _cases():
    out = []
    for fmt in ("nvfp4", "mxfp4"):
        for M, layer in ((1, 0), (64, 0), (2048, 31)):
            out += [p for p in config_problems(5, M=M, fmt=fmt) if p.extra["layer"] == layer]
        out += [p for p in config_problems(5, M=8192, fmt=fmt)
                if p.extra["layer"] == 7 and p.extra["idx"] in (4, 6)]  # gate, down
    return out


CASES = sorted(_cases(), key=lambda p: (p.extra["w_seed"], p.fmt, p.M))


_W = {}  # weights of one linear are shared by its row counts and formats


def _make(prob):
    key = (prob.extra["w_seed"], prob.K, prob.N)
    if key not in _W:
        _W.clear()
        _W[key] = prob.make()[1]
    return prob.make_x(), _W[key]


@pytest.mark.parametrize("prob", CASES, ids=[f"{p.fmt}-{p.name}" for p in CASES])
def test_stack_linear_sampled(prob):
    import fp4_sparse_dense_b200 as sq
    import torch
    x, w = _make(prob)
    cfg = cfg_of(prob.fmt, "pair48")
    act = sq.prepare(to_device(x), cfg)
    wt = sq.quantize_weight(to_device(w), cfg)
    y = sq.linear(act, wt).float().cpu().numpy()
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    rng = np.random.default_rng(prob.seed + prob.extra["w_seed"])
    M, N = prob.M, prob.N
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(M, 12), replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 96, replace=False)]))
    amax_x = S.amax_of(x.values) if prob.fmt == "nvfp4" else None
    amax_w = S.amax_of(w.values) if prob.fmt == "nvfp4" else None
    p = S.prepare(x.values[rows], prob.fmt, "pair48", amax=amax_x)
    qw = S.quantize_weight(w.values[:, cols], prob.fmt, "pair48", amax=amax_w)
    y64 = S.linear(p, qw)
    assert rel_fro(y[np.ix_(rows, cols)], F.bf16_round(y64)) <= TOL_BF16
    # prepared backbone codes of the sampled rows, bit-exact (compressed rows are K/4 bytes)
    bq = act.bq[: M * prob.K // 4].view(M, prob.K // 4).cpu().numpy()
    assert np.array_equal(bq[rows], S.act_buffers(p)["bq"].reshape(len(rows), -1))


def test_stack_covers_every_linear_shape():
    shapes = {(p.K, p.N) for p in CASES}
    assert shapes == {(k, n) for _, k, n in LLAMA8B_LINEARS}
    assert {p.fmt for p in CASES} == {"nvfp4", "mxfp4"}
