#!/usr/bin/env python
"""Benchmark of the SharQ sparse-dense FP4 linear layer on B200.

One step = the whole hot path on one batch: activation preparation (tensor amax pass +
fused mask / FP4 quantisation / residual / metadata kernel) and the fused sparse + dense
FP4 GEMM with its bf16 epilogue. The weight is quantised once, before timing (it is an
offline step). Inputs are seeded synthetic tensors with the workloads' shapes and value
distributions (workloads/), resident in HBM before the timed region; several input sets
rotate so that every step reads operands that are not in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mlp_gate_up]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun): every rank runs its own batch (independent token batches, no
collective on the data path); value = all ranks' FLOPs / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SharQ linear TFLOPS (2MNK/t) and % FP4 peak; prep kernel HBM GB/s"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
NOMINAL_FP4_TFLOPS = 9000.0  # B200 dense FP4, spec sheet (context only)
NOMINAL_HBM_GBS = 7700.0     # B200 HBM3e, HGX spec sheet (context only)
L2_BYTES = 126 * 2**20  # B200 L2


def prep_bytes_per_elem(fmt: str, mask: str, residual: bool) -> float:
    """Algorithmic HBM bytes per X element of the preparation: the 16-bit read plus every
    output (codes, scales, metadata); the pair-wise backbone is stored compressed."""
    rb = 16 if fmt == "nvfp4" else 32
    pair = mask.startswith("pair48")
    b = 2.0 + (0.25 if pair else 0.5) + 1.0 / (32 if pair else rb)
    b += {"pair48": 1 / 16, "pair48_given": 0.0, "elem24": 1 / 8, "none": 0.0}[mask]
    if residual:
        b += 0.5 + 1.0 / rb
    return b


def metric_ceiling(mask: str, residual: bool) -> float:
    """2MNK / t at full tensor-pipe use, as a fraction of the dense FP4 peak: the sparse MMA
    runs the backbone's 2MNK at twice the dense rate, the dense MMAs at the dense rate."""
    t = (0.5 if mask.startswith("pair48") else 1.0) + (1.0 if residual else 0.0)
    return 1.0 / t


def prep_kernels(fmt: str, mask: str, residual: str = "on", given_amax: bool = False) -> list:
    if given_amax:  # the caller's NVFP4 amax: one kernel with the mask inline
        return ["prep_pair_kernel"]
    if mask.startswith("pair48"):
        # the residual's own tensor scale runs the quantisation twice (amax|r| in between)
        quant = ["prep_pair_kernel"] * (2 if residual == "own" else 1)
        return (["prep_mask_kernel"] if fmt == "nvfp4" else []) + quant
    return (["amax_kernel"] if fmt == "nvfp4" else []) + ["prep_elem_kernel"]


WORKLOADS = {
    # name: (M, K, N, per_row_outliers)
    "mlp_gate_up": (4096, 4096, 14336, False),
    "attn_proj": (2048, 4096, 4096, False),
    "mlp_down": (4096, 14336, 4096, True),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _code_only(text: str) -> str:
    """C++ source without comments and blank space (a comment edit leaves the code, and so
    the kernels the counters were taken on, unchanged)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def src_hash(files):
    h = hashlib.sha1()
    for f in files:
        h.update(_code_only(open(os.path.join(ROOT, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:12]


GEMM_SRC = ["fp4_sparse_dense_b200/csrc/gemm.cu", "fp4_sparse_dense_b200/csrc/gemm_pair.cu",
            "fp4_sparse_dense_b200/csrc/epilogue.cuh", "fp4_sparse_dense_b200/csrc/sm100_ptx.cuh",
            "fp4_sparse_dense_b200/csrc/sharq_internal.h"]


def gemm_kernel_name(M: int, N: int, residual: str = "on") -> str:
    """Which GEMM kernel sharq_linear launches for this shape (CTA pair for M >= 256; the
    two-accumulator variant of the residual's own scale always runs the one-CTA kernel)."""
    pair = M >= 256 and N % 256 == 0 and residual != "own"
    return "sharq_gemm_pair_kernel" if pair else "sharq_gemm_kernel"


def traffic_from_profile(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary, when it was taken on the
    current GEMM source (else None)."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload)
    if not e or e.get("gemm_src") != src_hash(GEMM_SRC):
        return None
    return e.get("dram_bytes_per_launch")


PREP_SRC = ["fp4_sparse_dense_b200/csrc/prep.cu", "fp4_sparse_dense_b200/csrc/fp4_quant.cuh",
            "fp4_sparse_dense_b200/csrc/fp4_device.cuh", "fp4_sparse_dense_b200/csrc/sm100_ptx.cuh",
            "fp4_sparse_dense_b200/csrc/sharq_internal.h"]


def prep_issue_from_profile(workload: str):
    """Warp instructions per X element of the preparation (all its kernels) from the
    committed ncu count, when it was taken on the current preparation source (else None)."""
    p = os.path.join(ROOT, "profiles", "prep_issue.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(workload)
    if not e or e.get("prep_src") != src_hash(PREP_SRC):
        return None
    return e.get("warp_instructions_per_elem")


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"sharq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        if not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w_max": max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
                if any(r[2].replace(".", "").isdigit() for r in rows) else None}


def rank_seed(rank: int) -> int:
    """Each rank draws its own token batch (independent problems, weak scaling)."""
    return 1000 + rank


def max_over_ranks(ms: float, dist_mod, device) -> float:
    """Elapsed device time of the slowest rank (every rank calls this, same order)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist_mod is not None and dist_mod.is_initialized() and dist_mod.get_world_size() > 1:
        dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, world: int, steps: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: all ranks' work divided by the slowest rank's time."""
    return flops_per_step * world * steps / (ms_max * 1e-3) / 1e12


def run_pipelined(n, slots, prep, gemm):
    """n items, the preparation of item j+1 on a side stream (launched to share the SMs,
    sharq_prepare_alongside) while the GEMMs of item j run on the current stream. prep(j, s)
    writes activation slot j % slots on stream s; gemm(j) reads it. A slot is rewritten only
    after the GEMMs that read it are done; the side stream joins the current one at the end."""
    import torch
    main = torch.cuda.current_stream()
    side = run_pipelined.side = getattr(run_pipelined, "side", None) or torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in range(slots)]
    done = [torch.cuda.Event() for _ in range(slots)]
    side.wait_stream(main)
    with torch.cuda.stream(side):
        prep(0, side)
        ready[0].record(side)
    for i in range(n):
        j = i + 1
        if j < n:
            with torch.cuda.stream(side):
                if j >= slots:
                    side.wait_event(done[j % slots])
                prep(j, side)
                ready[j % slots].record(side)
        main.wait_event(ready[i % slots])
        gemm(i)
        done[i % slots].record(main)
    main.wait_stream(side)


def input_sets(M: int, K: int, N: int) -> int:
    """Input sets (X, its prepared buffers and Y) the timed steps rotate over: at least 3,
    and enough that one rotation's X and Y exceed 2.5x the L2, so that no step finds its
    operands in L2 from the previous rotation. Decode-sized M rotates its weights instead."""
    if M < 256:
        return 3
    return max(3, -(-int(2.5 * L2_BYTES) // (M * K * 2 + M * N * 2)))


def weight_bytes(qw):
    """Bytes of a quantised weight the GEMM reads: codes and both scale views."""
    return sum(b.numel() * b.element_size() for b in (qw.codes, qw.scales_dense, qw.scales_sparse)
               if b is not None)


def act_tensors(a):
    """The device buffers of a prepared activation (None where the configuration has none)."""
    return [t for t in (a.bq, a.bs, a.bm, a.rq, a.rs) if t is not None]


def workload_shape(args):
    """(M, K, N) of a single-linear workload; --m replaces its token rows (decode sizes)."""
    M, K, N, _ = WORKLOADS[args.workload]
    return (args.m if args.m else M), K, N


def make_inputs(workload: str, seed: int, M: int = None):
    from workloads import gaussian_weight, heavy_activations
    M0, K, N, per_row = WORKLOADS[workload]
    M = M or M0
    rng = np.random.default_rng(seed)
    x = heavy_activations(rng, M, K, per_row=per_row)
    w = gaussian_weight(rng, K, N)
    return x, w


def oracle_modes(args) -> dict:
    """prepare() keyword arguments of the oracle for the bench's --fmt/--mask/--residual."""
    kw = {"fmt": args.fmt, "mask": args.mask, "residual": args.residual != "off"}
    if args.residual == "unquantized":
        kw["residual_ref"] = "unquantized"
    if args.residual == "own":  # amax|r| over each sampled block of rows
        kw["residual_scale"] = "own"
    return kw


def cpu_baseline(workload: str, budget_s: float, x, qw, kw=None):
    """The oracle as it stands, on a bounded sample: blocks of 16 token rows prepared and
    multiplied by the whole weight (quantised beforehand: an offline step) until the
    budget of CPU time is used. Returns (TFLOP/s, cores, sample description)."""
    from oracle import sharq as S
    kw = dict(kw or {})
    _, K, N, _ = WORKLOADS[workload]
    M = x.values.shape[0]
    amax = S.amax_of(x.values) if kw.get("fmt", "nvfp4") == "nvfp4" else None
    given = None
    if kw.get("mask") == S.PAIR48_GIVEN:
        given = S.static_keep_pairs48(x.values, 16)
    rows = 16
    t_used, n_rows = 0.0, 0
    while t_used < budget_s and n_rows < M:
        t0 = time.perf_counter()
        xs = x.values[n_rows:n_rows + rows]
        p = S.prepare(xs, amax=amax, given=None if given is None else given[: len(xs)], **kw)
        S.linear(p, qw)
        t_used += time.perf_counter() - t0
        n_rows += len(xs)
    flops = 2.0 * n_rows * N * K
    cores = len(os.sched_getaffinity(0))
    return flops / t_used / 1e12, cores, f"{n_rows} of {M} rows x all {N} columns, K={K}; " \
        f"{t_used:.1f} s of CPU work (weight quantised beforehand)"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload not in WORKLOADS:
        raise SystemExit("the reference arm times the single-linear workloads "
                         f"({', '.join(WORKLOADS)})")
    from oracle import sharq as S
    M, K, N = workload_shape(args)
    x, w = make_inputs(args.workload, rank_seed(0), M)
    kw = oracle_modes(args)
    qw = S.quantize_weight(w.values, args.fmt, args.mask)  # offline, outside the samples
    budget = max(1.0, 90.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(args.workload, budget, x, qw, kw)
    vals = []
    for _ in range(args.steps):
        v, cores, sample = cpu_baseline(args.workload, budget, x, qw, kw)
        vals.append(v)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 2.0 * M * N * K / (value * 1e12) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "format": args.fmt,
                   "mask": args.mask, "residual": args.residual},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import fp4_sparse_dense_b200 as sq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    M, K, N = workload_shape(args)
    res_mode = {"on": True, "off": False, "unquantized": "unquantized", "own": "own"}[args.residual]
    cfg = sq.Config.from_names(args.fmt, args.mask, res_mode)  # default: the method
    has_res = args.residual != "off"

    x16, w16 = make_inputs(args.workload, rank_seed(rank), M)
    from workloads import to_device
    n_sets = input_sets(M, K, N)
    X = [to_device(x16, dev) for _ in range(n_sets)]
    W = [to_device(w16, dev) for _ in range(2)]
    QW = [sq.quantize_weight(w, cfg) for w in W]
    wbytes = weight_bytes(QW[0])
    decode = M < 256  # the weight stream dominates: rotate enough copies to stream from HBM
    if decode:
        QW += [sq.quantize_weight(W[j % 2], cfg) for j in range(2, -(-int(2.5 * L2_BYTES) // wbytes))]
    n_w = len(QW)
    ACT = [sq.empty_act(M, K, cfg, dev) for _ in range(n_sets)]
    Y = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(n_sets)]
    if args.mask == "pair48_given":
        # ablation set-up (outside the timed region): a static mask, the pair mask of the
        # per-column max |x| of the first input set, replicated to every row in the PAIR
        # metadata layout ([K/256 slices][rows padded to 128][16 bytes], padding 0x44)
        col = X[0].abs().amax(dim=0, keepdim=True).to(X[0].dtype)
        one = sq.prepare(col, sq.Config.from_names(args.fmt, "pair48", False))
        KS, Mp = K // 256, (M + 127) // 128 * 128
        row0 = one.bm.view(KS, 128, 16)[:, :1, :]
        full = torch.full((KS, Mp, 16), 0x44, dtype=torch.uint8, device=dev)
        full[:, :M, :] = row0
        for a in ACT:
            a.bm[: full.numel()].copy_(full.view(-1))
    WS = sq.linear_workspace(M, N, K, cfg, dev)  # split-K scratch (None for prefill shapes)
    stream = torch.cuda.current_stream()

    # --given-amax: the NVFP4 tensor amax of each input set reduced beforehand (outside the
    # timed region, by torch) and passed in; the preparation is then a single kernel
    AMX = [x.abs().max().float().reshape(1) for x in X] if args.given_amax else [None] * n_sets

    def step(i):
        a = sq.prepare(X[i % n_sets], cfg, out=ACT[i % n_sets], amax=AMX[i % n_sets])
        return a

    for i in range(args.warmup):
        sq.linear(step(i), QW[i % n_w], out=Y[i % n_sets], workspace=WS)
    torch.cuda.synchronize()
    status = sq.sharq_device_status()
    assert status == 0, sq.sharq_status_string(status)

    # the timed region: K whole steps back to back, no host work or events between kernels
    # (an event between the two calls would hold back the GEMM's programmatic early launch)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    def timed_steps(k):
        if args.pipeline:
            run_pipelined(k, n_sets,
                          lambda j, s: sq.prepare(X[j % n_sets], cfg, out=ACT[j % n_sets],
                                                  stream=s, alongside=True),
                          lambda j: sq.linear(ACT[j % n_sets], QW[j % n_w], out=Y[j % n_sets],
                                              workspace=WS))
        else:
            for i in range(k):
                sq.linear(step(i), QW[i % n_w], out=Y[i % n_sets], workspace=WS)

    if args.pipeline:  # warm the two-stream schedule too
        timed_steps(args.warmup)
        torch.cuda.synchronize()
    with Clocks(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        timed_steps(args.steps)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    ms_max = max_over_ranks(ms, dist, dev)

    # per-kernel durations for the roofline: a second pass with events around each call on
    # the launching stream
    n_ev = min(args.steps, 200)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_ev)]
    for i in range(n_ev):
        ev[i][0].record(stream)
        a = step(i)
        ev[i][1].record(stream)
        sq.linear(a, QW[i % n_w], out=Y[i % n_sets], workspace=WS)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    prep_ms = [e[0].elapsed_time(e[1]) for e in ev]
    gemm_ms = [e[1].elapsed_time(e[2]) for e in ev]

    # the preparation alone, calls back to back (as in a layer, where each one's launch hides
    # behind the previous kernel) over enough input sets that every call reads X from HBM
    xb = M * K * 2 + sum(t.numel() * t.element_size() for t in act_tensors(ACT[0]))
    n_prep = max(2, -(-int(2.5 * L2_BYTES) // xb))
    if decode:  # a few rows of X fit in L2 whatever we do; 64 sets bound the set-up
        n_prep = min(n_prep, 64)
    XP = [X[j % n_sets] if j < n_sets else torch.empty_like(X[0]).copy_(X[j % n_sets])
          for j in range(n_prep)]
    AMP = [AMX[j % n_sets] for j in range(n_prep)]
    AP = [ACT[j] if j < n_sets else sq.empty_act(M, K, cfg, dev) for j in range(n_prep)]
    if args.mask == "pair48_given":
        for a in AP[n_sets:]:
            a.bm.copy_(ACT[0].bm)
    n_pc = max(3 * n_prep, min(args.steps, 200))
    for j in range(n_prep):
        sq.prepare(XP[j], cfg, out=AP[j], amax=AMP[j])
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for j in range(n_pc):
        sq.prepare(XP[j % n_prep], cfg, out=AP[j % n_prep], amax=AMP[j % n_prep])
    p1.record(stream)
    torch.cuda.synchronize()
    prep_b2b = p0.elapsed_time(p1) / n_pc
    del XP, AP
    flops = 2.0 * M * N * K
    value = job_throughput(flops, world, args.steps, ms_max)

    # end to end through the public API with host buffers (pinned), copies timed: every step
    # copies its X in and its Y out. The copies run on their own streams (one per
    # direction, so PCIe carries both at once) and overlap the neighbouring steps' compute;
    # a buffer set is reused only after the copy and the compute that use it are done.
    xh = [X[i].cpu().pin_memory() for i in range(n_sets)]
    yh = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(n_sets)]
    e2e_steps = max(1, min(args.steps, 30))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_sets)]
    ev_done = [torch.cuda.Event() for _ in range(n_sets)]
    ev_out = [torch.cuda.Event() for _ in range(n_sets)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(e2e_steps):
        j = i % n_sets
        with torch.cuda.stream(s_in):
            if i >= n_sets:
                s_in.wait_event(ev_done[j])  # step i - n_sets has read X[j]
            X[j].copy_(xh[j], non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= n_sets:
            stream.wait_event(ev_out[j])  # Y[j] of step i - n_sets has been copied out
        a = step(i)
        sq.linear(a, QW[i % n_w], out=Y[j], workspace=WS)
        ev_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            yh[j].copy_(Y[j], non_blocking=True)
            ev_out[j].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_value = job_throughput(flops, world, e2e_steps,
                               max_over_ranks(e0.elapsed_time(e1), dist, dev))
    status = sq.sharq_device_status()
    assert status == 0, sq.sharq_status_string(status)

    if rank == 0:
        hbm, bf16, bf16_sus, peak_src = load_peaks()
        fp4_peak = bf16_sus * FP4_OVER_BF16
        gemm_avg = float(np.mean(gemm_ms))
        prep_avg = prep_b2b
        prep_in_step = float(np.mean(prep_ms))
        gemm_tflops = flops / (gemm_avg * 1e-3) / 1e12
        bpe = prep_bytes_per_elem(args.fmt, args.mask, has_res)
        prep_gbs = M * K * bpe / (prep_avg * 1e-3) / 1e9
        # the committed capture is of the method's kernel (NVFP4, pair 4:8, residual on)
        method = ((args.fmt, args.mask, args.residual) == ("nvfp4", "pair48", "on")
                  and not args.given_amax and M == WORKLOADS[args.workload][0])
        traffic = traffic_from_profile(args.workload) if method else None
        clocks = clk.summary()
        # the preparation is bound by instruction issue, not HBM: its issue-rate roofline
        # (warp instructions per element from the committed count; peak = 4 issues per SM
        # per cycle at the median SM clock of the timed region)
        ipe = prep_issue_from_profile(args.workload) if method else None
        issue = None
        if ipe and clocks.get("sm_mhz"):
            n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
            peak_i = n_sm * 4 * clocks["sm_mhz"] * 1e6
            ach_i = ipe * M * K / (prep_avg * 1e-3)
            issue = {"warp_instructions_per_elem": ipe, "achieved_ginst_s": ach_i / 1e9,
                     "peak_ginst_s": peak_i / 1e9, "frac": ach_i / peak_i,
                     "peak_source": f"{n_sm} SMs x 4 issue slots x {clocks['sm_mhz']} MHz"}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4",
            "data": "synthetic",
            "config": {"workload": args.workload, "M": M, "K": K, "N": N, "format": args.fmt,
                       "mask": args.mask, "residual": args.residual, "out": "bf16",
                       "l2": (f"weights rotate over {n_w} copies ({n_w * wbytes / 1e6:.0f} MB "
                              "> 126 MB L2)") if decode else
                             (f"{n_sets} rotating input sets ({n_sets * (M * K + M * N) * 2 / 1e6:.0f}"
                              " MB of X and Y > 126 MB L2)"),
                       "schedule": ("pipelined: step i+1's preparation beside step i's GEMM "
                                    "(two streams)") if args.pipeline else "serial",
                       "amax": "given (reduced before the timed region)" if args.given_amax
                               else "reduced in every call",
                       "parallelism": f"dp{world}"},
            "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                         "traffic": traffic,
                         "peak_source": f"{peak_src}: bf16 sustained {bf16_sus} x "
                                        f"{FP4_OVER_BF16} (nominal FP4:BF16)",
                         "ceiling_frac": metric_ceiling(args.mask, has_res),
                         # the tensor pipe's executed work (sparse backbone at twice the
                         # dense rate): 2MNK / ceiling per launch, against the same peak
                         "executed_frac": gemm_tflops / fp4_peak / metric_ceiling(args.mask, has_res),
                         # against 4x the measured bf16 burst figure instead of the sustained
                         "frac_vs_burst_peak": gemm_tflops / (bf16 * FP4_OVER_BF16),
                         # context: the spec sheet's dense FP4 figure
                         "frac_vs_nominal_peak": gemm_tflops / NOMINAL_FP4_TFLOPS,
                         "kernel": gemm_kernel_name(M, N, args.residual), "kernel_ms": gemm_avg},
            "prep": {"ms": prep_avg, "gbs": prep_gbs, "hbm_peak_gbs": hbm,
                     "frac": prep_gbs / hbm,
                     "frac_vs_nominal_hbm": prep_gbs / NOMINAL_HBM_GBS,
                     "bytes_per_elem": bpe,
                     "ms_in_step": prep_in_step,
                     "issue_roofline": issue,
                     "kernel": " + ".join(prep_kernels(args.fmt, args.mask, args.residual,
                                                       args.given_amax)),
                     "note": ("ms: calls back to back over "
                              + ("input sets larger than L2 (X read from HBM every call)"
                                 if n_prep * xb >= 2 * L2_BYTES else
                                 f"{n_prep} input sets (a few rows: X stays in L2)")
                              + "; ms_in_step: between events around the call inside the "
                                "step, which adds the first kernel's launch gap; algorithmic "
                                "bytes count X once")},
            "gemm_tflops": gemm_tflops,
            "pct_fp4_peak": 100.0 * gemm_tflops / fp4_peak,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": M * K * 2,
                    "d2h_bytes_per_step": M * N * 2},
            "gpu_launches": (len(prep_kernels(args.fmt, args.mask, args.residual,
                                              args.given_amax)) + 1 +
                             (1 if WS is not None else 0)) * args.steps,
            "clocks": clocks,
        }
        if decode:  # below the ridge point the GEMM streams its weight: an HBM roofline
            gbs = wbytes / (gemm_avg * 1e-3) / 1e9
            line["roofline"] = {
                "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "traffic": None, "peak_source": f"{peak_src}: copy bandwidth",
                "note": "FP4 weight payload (codes and both scale views) / linear call time "
                        "(split-K partials summed by a second kernel when the workspace is used)",
                "weight_bytes": wbytes, "split_k": WS is not None,
                "kernel": gemm_kernel_name(M, N, args.residual), "kernel_ms": gemm_avg}
        if not args.no_cpu_baseline and world == 1:
            from oracle import sharq as S
            qw_cpu = S.quantize_weight(w16.values, args.fmt, args.mask)
            v, cores, sample = cpu_baseline(args.workload, args.cpu_budget, x16, qw_cpu,
                                            oracle_modes(args))
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores,
                                    "kind": "oracle", "sample": sample}
            # the same oracle held to one thread (numpy's BLAS pool limited to 1)
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    v1, _, sample1 = cpu_baseline(args.workload, args.cpu_budget / 3, x16,
                                                  qw_cpu, oracle_modes(args))
                line["cpu_baseline"]["one_thread"] = {"value": v1, "unit": "TFLOP/s",
                                                      "sample": sample1}
            except ImportError:
                pass
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_stack(args):
    """One Llama-3-8B-shaped layer per step (config 5): q, k, v share one preparation of the
    attention input, o has its own, gate and up share the MLP input's, down has its own.
    Weights rotate over 4 layers (436 MB of FP4 payload), so a step streams its weights from
    HBM as a model's would. Inputs are synthetic (drawn on the device, outlier channels per
    row); they are not chained from layer to layer (there are no norms between them here)."""
    import torch
    import fp4_sparse_dense_b200 as sq
    from workloads import LLAMA8B_LINEARS
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    M = args.m or 1
    cfg = sq.Config.from_names(args.fmt, args.mask,
                               {"on": True, "off": False, "unquantized": "unquantized",
                                "own": "own"}[args.residual])
    g = torch.Generator(device=dev).manual_seed(5000 + M)
    shapes = {nm: (k, n) for nm, k, n in LLAMA8B_LINEARS}
    groups = [("attn", 4096, ["q", "k", "v"]), ("o", 4096, ["o"]), ("mlp", 4096, ["gate", "up"]),
              ("down", 14336, ["down"])]
    if args.fused:  # deployment layout: q|k|v and gate|up weights concatenated along N
        shapes = {"qkv": (4096, 6144), "o": (4096, 4096), "gate_up": (4096, 28672),
                  "down": (14336, 4096)}
        groups = [("attn", 4096, ["qkv"]), ("o", 4096, ["o"]), ("mlp", 4096, ["gate_up"]),
                  ("down", 14336, ["down"])]
    layers = 4

    def act_input(K):
        x = torch.randn(M, K, device=dev, generator=g)
        out = torch.rand(M, K, device=dev, generator=g) < 0.005
        gain = 20 + 30 * torch.rand(M, K, device=dev, generator=g)
        return torch.where(out, x * gain, x).to(torch.bfloat16)

    X = {gname: act_input(K) for gname, K, _ in groups}
    A = {gname: sq.empty_act(M, K, cfg, dev) for gname, K, _ in groups}
    QW = []
    for _ in range(layers):
        lw = {}
        for nm, (k, n) in shapes.items():
            w = (torch.randn(k, n, device=dev, generator=g) * 0.02).to(torch.bfloat16)
            lw[nm] = sq.quantize_weight(w, cfg)
            del w
        QW.append(lw)
    Y = {nm: torch.empty(M, n, dtype=torch.bfloat16, device=dev) for nm, (k, n) in shapes.items()}
    WS = {nm: sq.linear_workspace(M, n, k, cfg, dev) for nm, (k, n) in shapes.items()}
    flops = sum(2.0 * M * k * n for k, n in shapes.values())
    wbytes = 0
    for t in (QW[0][nm] for nm in shapes):
        wbytes += sum(b.numel() for b in (t.codes, t.scales_dense, t.scales_sparse) if b is not None)

    def layer(i):
        lw = QW[i % layers]
        for gname, _, names in groups:
            a = sq.prepare(X[gname], cfg, out=A[gname])
            for nm in names:
                sq.linear(a, lw[nm], out=Y[nm], workspace=WS[nm])

    ng = len(groups)

    def layers_run(k):
        if args.pipeline:  # group t+1's preparation beside group t's GEMMs, across layers
            def prep(t, s):
                gname, _, _ = groups[t % ng]
                sq.prepare(X[gname], cfg, out=A[gname], stream=s, alongside=True)

            def gemms(t):
                gname, _, names = groups[t % ng]
                lw = QW[(t // ng) % layers]
                for nm in names:
                    sq.linear(A[gname], lw[nm], out=Y[nm], workspace=WS[nm])
            run_pipelined(k * ng, ng, prep, gemms)
        else:
            for i in range(k):
                layer(i)

    layers_run(args.warmup)
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    graph = None
    if args.graph:
        # one CUDA graph of `layers` layers (every weight set once): replaying it launches
        # the same kernels with the same programmatic dependencies, without the host calls
        if args.steps % layers:
            args.steps += layers - args.steps % layers
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layers_run(layers)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        assert sq.sharq_device_status() == 0
    stream = torch.cuda.current_stream()
    with Clocks(0) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if graph is not None:
            for _ in range(args.steps // layers):
                graph.replay()
        else:
            layers_run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert sq.sharq_device_status() == 0
    per_layer_ms = ms / args.steps
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    value = flops * args.steps / (ms * 1e-3) / 1e12
    hbm_bound = M < 256  # weight stream dominates below the ridge point (~850 flop/byte)
    achieved = (wbytes / (per_layer_ms * 1e-3) / 1e9) if hbm_bound else value
    peak = hbm if hbm_bound else bf16_sus * FP4_OVER_BF16
    n_prep = sum(len(prep_kernels(args.fmt, args.mask, args.residual)) for _ in groups)
    n_gemm = sum(1 + (1 if WS[nm] is not None else 0) for nm in shapes)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_layer_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp4",
        "data": "synthetic (drawn on the device)",
        "config": {"workload": "stack8b", "M": M, "fused": bool(args.fused),
                   "schedule": "pipelined" if args.pipeline else "serial",
                   "launch": f"CUDA graph of {layers} layers" if args.graph else "eager",
                   "linears": [f"{nm} {k}x{n}" for nm, (k, n) in shapes.items()],
                   "layers_rotated": layers, "format": args.fmt, "mask": args.mask,
                   "residual": args.residual, "out": "bf16",
                   "l2": f"weights rotate over {layers} layers ({layers * wbytes / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": "dp1"},
        "roofline": {"bound": "hbm" if hbm_bound else "tensor", "achieved": achieved, "peak": peak,
                     "unit": "GB/s" if hbm_bound else "TFLOP/s", "frac": achieved / peak,
                     "traffic": None,
                     "note": ("FP4 weight payload (codes and both scale views) per layer / layer "
                              "time" if hbm_bound else "2MNK of the 7 linears / layer time"),
                     "weight_bytes_per_layer": wbytes},
        "gpu_launches": (n_prep + n_gemm) * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="sharq", choices=["sharq", "reference"])
    ap.add_argument("--workload", default="mlp_gate_up", choices=list(WORKLOADS) + ["stack8b"])
    ap.add_argument("--m", type=int, default=None,
                    help="token rows: of --workload stack8b (default 1), or replacing a "
                         "single-linear workload's M (decode sizes)")
    ap.add_argument("--fused", action="store_true",
                    help="stack8b: q|k|v and gate|up weights concatenated (4 GEMMs per layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pipeline", action="store_true",
                    help="two streams: the next step's (stack8b: group's) preparation runs "
                         "beside the current GEMM (sharq_prepare_alongside)")
    ap.add_argument("--given-amax", action="store_true",
                    help="NVFP4 pair mask: pass each input's tensor amax, reduced beforehand "
                         "(sharq_prepare_given_amax), instead of reducing it in every call")
    ap.add_argument("--graph", action="store_true",
                    help="stack8b: replay the layers from one CUDA graph (no host calls in the "
                         "timed region)")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"])
    ap.add_argument("--mask", default="pair48",
                    choices=["pair48", "elem24", "pair48_given", "none"],
                    help="pair48 is the method; the others are ablations / baselines "
                         "(none with --residual off: plain FP4)")
    ap.add_argument("--residual", default="on", choices=["on", "off", "unquantized", "own"],
                    help="own: the residual with its own tensor scale (two accumulators)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "stack8b":
        return run_stack(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
