#!/usr/bin/env python
"""Benchmark of the SharQ sparse-dense FP4 linear layer on B200.

One step = the whole hot path on one batch. The default workload is the 8B-shaped layer
(the seven Llama-3-8B linears; q|k|v and gate|up concatenated along N, the deployment
layout) at M = 8192 token rows: four activation preparations (tensor amax, pair mask, FP4
backbone and residual, metadata) and four fused sparse + dense FP4 GEMMs with their bf16
epilogues. Single linears (--workload mlp_gate_up / attn_proj / mlp_down) are the other
workloads. Weights are quantised once, before timing (an offline step). Inputs are seeded
synthetic tensors with the workloads' shapes and value distributions, resident in HBM
before the timed region, and larger than L2 (or rotated so that no step finds its operands
in L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stack8b] [--m 8192]
    python bench.py --impl reference ...   # the CPU oracle on bounded samples

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
STACK_M = 8192  # default token rows of the 8B-shaped layer: the largest prefill of the sweep


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


def sustained_clock_mhz():
    """Median SM clock under which the sustained bf16 figure was measured (None if unknown)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return None
    return json.load(open(p)).get("clocks_under_load", {}).get("sm_mhz_median")


def fp4_peak(sm_mhz=None, sm_max_mhz=None):
    """Dense FP4 tensor peak for the GEMM roofline, taken at the clock of the timed region
    (sm_mhz: its median SM clock from the samples). A burst at full clock (the default short
    run) is held to 4 x the measured bf16 BURST figure; the sustained figure, taken at a lower
    clock under the power cap, would flatter it. A run long enough to sit under the power cap
    (median below 90 % of the maximum clock) is held to 4 x the sustained figure scaled from
    its own median clock to the run's. Returns (TFLOP/s, source)."""
    _, bf16, bf16_sus, src = load_peaks()
    sus_mhz = sustained_clock_mhz()
    if sm_mhz and sm_max_mhz and sus_mhz and sm_mhz < 0.9 * sm_max_mhz:
        peak = bf16_sus * (sm_mhz / sus_mhz) * FP4_OVER_BF16
        return peak, (f"{src}: bf16 sustained {bf16_sus} (at {sus_mhz:.0f} MHz) scaled to this "
                      f"run's median {sm_mhz:.0f} MHz x {FP4_OVER_BF16} (nominal FP4:BF16): the "
                      f"timed region ran under the power cap; context: x burst {bf16} = "
                      f"{bf16 * FP4_OVER_BF16:.1f}")
    return bf16 * FP4_OVER_BF16, (f"{src}: bf16 burst {bf16} x {FP4_OVER_BF16} (nominal FP4:BF16); "
                                  f"context: x sustained {bf16_sus} = {bf16_sus * FP4_OVER_BF16:.1f}")


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
    """DRAM bytes per GEMM launch from the committed ncu record, when it was taken on the
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


def prep_traffic_from_profile(workload: str):
    """DRAM bytes (read + write) per preparation call, all its kernels, from the committed
    ncu record, when it was taken on the current preparation source (else None)."""
    p = os.path.join(ROOT, "profiles", "prep_traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(workload)
    if not e or e.get("prep_src") != src_hash(PREP_SRC):
        return None
    return e.get("dram_bytes_per_call")


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


# the 8B-shaped layer's CPU sample: rows of every linear's input x columns of its weight
STACK_CPU_ROWS = 16
STACK_CPU_COLS = 512


def stack_layout(unfused: bool = False):
    """Linears of the 8B-shaped layer: ({name: (K, N)}, [(group, K, [names])]), a group being
    the linears that share one prepared input. Default: the deployment layout, q|k|v and
    gate|up concatenated along N (four GEMMs); unfused: the seven linears."""
    from workloads import LLAMA8B_LINEARS
    if unfused:
        shapes = {nm: (k, n) for nm, k, n in LLAMA8B_LINEARS}
        groups = [("attn", 4096, ["q", "k", "v"]), ("o", 4096, ["o"]),
                  ("mlp", 4096, ["gate", "up"]), ("down", 14336, ["down"])]
    else:
        shapes = {"qkv": (4096, 6144), "o": (4096, 4096), "gate_up": (4096, 28672),
                  "down": (14336, 4096)}
        groups = [("attn", 4096, ["qkv"]), ("o", 4096, ["o"]), ("mlp", 4096, ["gate_up"]),
                  ("down", 14336, ["down"])]
    return shapes, groups


def stack_cpu_samples(shapes, groups, x_rows, amax_x, w_cols, amax_w, kw):
    """Oracle operands of the layer's CPU sample: per linear the sampled input rows with the
    input's tensor amax, and the weight's sampled columns quantised (offline, untimed) with
    the weight's tensor amax. x_rows / amax_x are keyed by group, w_cols / amax_w by linear."""
    from oracle import sharq as S
    out = []
    for gname, K, names in groups:
        for nm in names:
            qw = S.quantize_weight(w_cols[nm], kw.get("fmt", "nvfp4"), kw.get("mask", "pair48"),
                                   amax=amax_w[nm])
            out.append({"name": nm, "x": x_rows[gname], "amax": amax_x[gname], "qw": qw,
                        "K": K, "cols": w_cols[nm].shape[1]})
    return out


def time_stack_passes(samples, budget_s, kw, min_passes=1):
    """The oracle as it stands over the layer's sample (every linear: prepare the sampled rows,
    multiply by the sampled weight columns), whole passes until the CPU-time budget is used.
    Returns (TFLOP/s, passes, seconds, rows per linear)."""
    from oracle import sharq as S
    kw = dict(kw)
    fmt = kw.get("fmt", "nvfp4")
    t_used, flops, passes = 0.0, 0.0, 0
    while passes < min_passes or t_used < budget_s:
        for smp in samples:
            t0 = time.perf_counter()
            p = S.prepare(smp["x"], amax=smp["amax"] if fmt == "nvfp4" else None, **kw)
            S.linear(p, smp["qw"])
            t_used += time.perf_counter() - t0
            flops += 2.0 * smp["x"].shape[0] * smp["cols"] * smp["K"]
        passes += 1
    return flops / t_used / 1e12, passes, t_used, samples[0]["x"].shape[0]


def reference_stack_samples(args, rank_seed_: int):
    """Synthetic sample of the 8B-shaped layer drawn on the host for the reference arm: the
    workloads' generator (Student-t rows, 0.5 % outlier channels redrawn per row; W ~
    N(0, 0.02)) for STACK_CPU_ROWS rows of every input and STACK_CPU_COLS columns of every
    weight. The tensor amaxes are those of the drawn samples (the full tensors are not drawn)."""
    from oracle import sharq as S
    from workloads import gaussian_weight, heavy_activations
    shapes, groups = stack_layout(args.unfused)
    rng = np.random.default_rng(rank_seed_)
    x_rows, amax_x, w_cols, amax_w = {}, {}, {}, {}
    for gname, K, _ in groups:
        x_rows[gname] = heavy_activations(rng, STACK_CPU_ROWS, K, per_row=True).values
        amax_x[gname] = S.amax_of(x_rows[gname])
    for nm, (k, n) in shapes.items():
        w_cols[nm] = gaussian_weight(rng, k, STACK_CPU_COLS).values
        amax_w[nm] = S.amax_of(w_cols[nm])
    return stack_cpu_samples(shapes, groups, x_rows, amax_x, w_cols, amax_w, oracle_modes(args))


def run_reference(args):
    """The CPU oracle as it stands, timed on the host's cores on bounded samples of the same
    workload (rank 0 only). Each step is one sample; ms_per_step is its real duration."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import sharq as S
    kw = oracle_modes(args)
    cores = len(os.sched_getaffinity(0))
    step_s, vals = [], []
    if args.workload == "stack8b":
        M = args.m or STACK_M
        shapes, _ = stack_layout(args.unfused)
        samples = reference_stack_samples(args, rank_seed(0))
        for _ in range(args.warmup):
            time_stack_passes(samples, 0.0, kw)
        for _ in range(args.steps):
            t0 = time.perf_counter()
            v, _, _, rows = time_stack_passes(samples, 0.0, kw)
            step_s.append(time.perf_counter() - t0)
            vals.append(v)
        sample = (f"per step {rows} rows x {STACK_CPU_COLS} columns of each of the "
                  f"{len(shapes)} linears ({', '.join(shapes)}), one pass; "
                  f"{args.steps} steps, {sum(step_s):.1f} s of CPU work in total")
        config = {"workload": "stack8b", "M": M, "fused": not args.unfused,
                  "linears": [f"{nm} {k}x{n}" for nm, (k, n) in shapes.items()],
                  "format": args.fmt, "mask": args.mask, "residual": args.residual}
    else:
        M, K, N = workload_shape(args)
        x, w = make_inputs(args.workload, rank_seed(0), M)
        qw = S.quantize_weight(w.values, args.fmt, args.mask)  # offline, outside the samples
        budget = max(1.0, 90.0 / max(1, args.steps + args.warmup))
        for _ in range(args.warmup):
            cpu_baseline(args.workload, budget, x, qw, kw)
        samples = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            v, cores, smp = cpu_baseline(args.workload, budget, x, qw, kw)
            step_s.append(time.perf_counter() - t0)
            vals.append(v)
            samples.append(smp)
        sample = (f"per step: {samples[0]}; {args.steps} steps, {sum(step_s):.1f} s of CPU "
                  "work in total")
        config = {"workload": args.workload, "M": M, "K": K, "N": N, "format": args.fmt,
                  "mask": args.mask, "residual": args.residual}
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * float(np.mean(step_s)), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def init_ranks():
    """(world, rank, local, device, dist) of this process; NCCL group when world > 1."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    return world, rank, local, torch.device("cuda", local), dist


def run_gpu(args, emit: bool = True, light: bool = False):
    """One single-linear workload. light: no end-to-end pass (used for the secondary line of
    the default run). Returns the JSON line (rank 0) and prints it when emit."""
    import torch
    import fp4_sparse_dense_b200 as sq

    world, rank, local, dev, dist = init_ranks()
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
    # Decode-sized steps (a few microseconds each) outrun the host's launches: they are
    # replayed from CUDA graphs (the same kernels with the same programmatic dependencies,
    # no host calls in the timed region), so the numbers are device time.
    use_graph = decode and not args.pipeline

    def captured(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        return g

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    g_steps = captured(lambda: timed_steps(args.steps)) if use_graph else None
    with Clocks(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        if g_steps is not None:
            g_steps.replay()
        else:
            timed_steps(args.steps)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    ms_max = max_over_ranks(ms, dist, dev)

    # per-kernel durations for the roofline: a second pass with events around each call on
    # the launching stream; for graph-replayed decode steps, a graph of the preparations
    # alone, the linear call's time being the rest of the step
    n_ev = min(args.steps, 200)
    if use_graph:
        del g_steps
        g_prep = captured(lambda: [step(i) for i in range(n_ev)])
        g_step = captured(lambda: timed_steps(n_ev))
        t_prep = timed(g_prep.replay) / n_ev
        t_step = timed(g_step.replay) / n_ev
        del g_prep, g_step
        prep_ms = [t_prep] * n_ev
        gemm_ms = [t_step - t_prep] * n_ev
    else:
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
    def prep_calls():
        for j in range(n_pc):
            sq.prepare(XP[j % n_prep], cfg, out=AP[j % n_prep], amax=AMP[j % n_prep])
    if use_graph:
        g_pc = captured(prep_calls)
        prep_b2b = timed(g_pc.replay) / n_pc
        del g_pc
    else:
        prep_b2b = timed(prep_calls) / n_pc
    del XP, AP
    flops = 2.0 * M * N * K
    value = job_throughput(flops, world, args.steps, ms_max)

    e2e_value = None
    if not light:
        e2e_value = e2e_single(args, stream, X, Y, QW, WS, n_sets, n_w, step, flops, world, dist,
                               dev)
    line = None
    if rank == 0:
        line = single_line(args, world, M, K, N, n_sets, n_w, wbytes, decode, WS, flops, value,
                           ms_max, gemm_ms, prep_b2b, prep_ms, n_prep, xb, e2e_value, clk, dev)
        if not args.no_cpu_baseline and world == 1 and not light:
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
        if emit:
            print(json.dumps(line), flush=True)
    if world > 1 and emit:
        dist.barrier()
        dist.destroy_process_group()
    return line


def e2e_single(args, stream, X, Y, QW, WS, n_sets, n_w, step, flops, world, dist, dev):
    """End to end through the public API with host buffers (pinned), copies timed: every step
    copies its X in and its Y out. The copies run on their own streams (one per direction,
    so PCIe carries both at once) and overlap the neighbouring steps' compute; a buffer set
    is reused only after the copy and the compute that use it are done."""
    import torch
    import fp4_sparse_dense_b200 as sq
    M, N = Y[0].shape
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
    return e2e_value


def single_line(args, world, M, K, N, n_sets, n_w, wbytes, decode, WS, flops, value, ms_max,
                gemm_ms, prep_b2b, prep_ms, n_prep, xb, e2e_value, clk, dev):
    """The JSON line of a single-linear workload (rank 0)."""
    import torch
    has_res = args.residual != "off"
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    clocks = clk.summary()
    peak, peak_source = fp4_peak(clocks.get("sm_mhz"), clocks.get("sm_max_mhz"))
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
                   "launch": ("steps replayed from a CUDA graph (decode-sized calls outrun "
                              "host launches)") if decode and not args.pipeline else "eager",
                   "amax": "given (reduced before the timed region)" if args.given_amax
                           else "reduced in every call",
                   "gemm_workspace": "split-K" if WS is not None else "none",
                   "parallelism": f"dp{world}"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": gemm_tflops / peak,
                     "traffic": traffic,
                     "peak_source": peak_source,
                     "ceiling_frac": metric_ceiling(args.mask, has_res),
                     # the tensor pipe's executed work (sparse backbone at twice the
                     # dense rate): 2MNK / ceiling per launch, against the same peak
                     "executed_frac": gemm_tflops / peak / metric_ceiling(args.mask, has_res),
                     # context: against 4x the sustained bf16 figure and the spec sheet
                     "frac_vs_sustained_peak": gemm_tflops / (bf16_sus * FP4_OVER_BF16),
                     "frac_vs_nominal_peak": gemm_tflops / NOMINAL_FP4_TFLOPS,
                     "kernel": gemm_kernel_name(M, N, args.residual), "kernel_ms": gemm_avg},
        "prep": {"ms": prep_avg, "gbs": prep_gbs, "hbm_peak_gbs": hbm,
                 "frac": prep_gbs / hbm,
                 "traffic": prep_traffic_from_profile(args.workload) if method else None,
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
        "pct_fp4_peak": 100.0 * gemm_tflops / peak,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * N * 2},
        # split-K (decode-sized M) adds a summing kernel
        "gpu_launches": (len(prep_kernels(args.fmt, args.mask, args.residual,
                                          args.given_amax)) + 1 +
                         (1 if WS is not None and decode else 0)) * args.steps,
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
    return line


def run_stack(args):
    """One Llama-3-8B-shaped layer per step: the attention input's preparation feeds q|k|v
    (or q, k, v), o has its own, gate|up (or gate, up) share the MLP input's, down has its
    own. Weights rotate over 4 layers (436 MB of FP4 payload), so a step streams its weights
    from HBM as a model's would. Inputs are synthetic, drawn on the device: Student-t(4) rows
    whose outlier channels (0.5 %, x U[20, 50]) are redrawn per row; they are not chained from
    layer to layer (there are no norms between them here). Under torchrun every rank runs its
    own batch (weak scaling)."""
    import torch
    import fp4_sparse_dense_b200 as sq
    world, rank, local, dev, dist = init_ranks()
    M = args.m or STACK_M
    cfg = sq.Config.from_names(args.fmt, args.mask,
                               {"on": True, "off": False, "unquantized": "unquantized",
                                "own": "own"}[args.residual])
    shapes, groups = stack_layout(args.unfused)
    layers = 4
    g = torch.Generator(device=dev).manual_seed(5000 + M + 7919 * rank)
    tdist = torch.distributions.StudentT(torch.tensor(4.0, device=dev))

    def act_input(K, idx):
        # StudentT draws from the global stream: one seed per input
        torch.manual_seed(5000 + M + 7919 * rank + 31 * idx)
        x = tdist.sample((M, K))
        out = torch.rand(M, K, device=dev, generator=g) < 0.005
        gain = 20 + 30 * torch.rand(M, K, device=dev, generator=g)
        return torch.where(out, x * gain, x).to(torch.bfloat16)

    cpu = (rank == 0 and world == 1 and not args.no_cpu_baseline)
    if cpu:  # the CPU baseline (rank 0, one GPU): the oracle's own amax of every full tensor
        from oracle import sharq as S
    cols = {nm: np.linspace(0, n - 1, STACK_CPU_COLS).astype(np.int64)
            for nm, (k, n) in shapes.items()}
    w_cols, amax_w = {}, {}
    X = {gname: act_input(K, i) for i, (gname, K, _) in enumerate(groups)}
    A = {gname: sq.empty_act(M, K, cfg, dev) for gname, K, _ in groups}
    QW = []
    for li in range(layers):
        lw = {}
        for nm, (k, n) in shapes.items():
            w = (torch.randn(k, n, device=dev, generator=g) * 0.02).to(torch.bfloat16)
            lw[nm] = sq.quantize_weight(w, cfg)
            if cpu and li == 0:  # the CPU baseline's weight sample (full-tensor amax)
                w_cols[nm] = w[:, torch.from_numpy(cols[nm]).to(dev)].float().cpu().numpy()
                amax_w[nm] = S.amax_of(w.float().cpu().numpy())
            del w
        QW.append(lw)
    Y = {nm: torch.empty(M, n, dtype=torch.bfloat16, device=dev) for nm, (k, n) in shapes.items()}
    WS = {nm: sq.linear_workspace(M, n, k, cfg, dev) for nm, (k, n) in shapes.items()}
    flops = sum(2.0 * M * k * n for k, n in shapes.values())
    lin_flops = {nm: 2.0 * M * k * n for nm, (k, n) in shapes.items()}
    wbytes = 0
    for t in (QW[0][nm] for nm in shapes):
        wbytes += sum(b.numel() for b in (t.codes, t.scales_dense, t.scales_sparse) if b is not None)
    stream = torch.cuda.current_stream()

    def layer(i, ev=None):
        """ev: ({group: (start, end)} around the preparations, {linear: end} after the GEMMs)."""
        lw = QW[i % layers]
        for gname, _, names in groups:
            if ev is not None:
                ev[0][gname][0].record(stream)
            a = sq.prepare(X[gname], cfg, out=A[gname])
            if ev is not None:
                ev[0][gname][1].record(stream)
            for nm in names:
                sq.linear(a, lw[nm], out=Y[nm], workspace=WS[nm])
                if ev is not None:
                    ev[1][nm].record(stream)

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
    if args.graph or M < 256:  # decode-sized layers outrun host launches: replay a graph
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
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if graph is not None:
            for _ in range(args.steps // layers):
                graph.replay()
        else:
            layers_run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, dist, dev)
    assert sq.sharq_device_status() == 0
    if graph is not None:
        del graph

    # per-kernel durations: a second pass with events around every call on the launching
    # stream (the first GEMM of a group then launches without its programmatic overlap)
    n_ev = max(1, min(args.steps, 50))
    evs = []
    for i in range(n_ev):
        ev = ({gname: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for gname, _, _ in groups},
              {nm: torch.cuda.Event(enable_timing=True) for nm in shapes})
        layer(i, ev)
        evs.append(ev)
    torch.cuda.synchronize()
    prep_ms = {gname: float(np.mean([e[0][gname][0].elapsed_time(e[0][gname][1]) for e in evs]))
               for gname, _, _ in groups}
    gemm_ms = {}
    for gname, _, names in groups:
        prev = [e[0][gname][1] for e in evs]
        for nm in names:
            gemm_ms[nm] = float(np.mean([p.elapsed_time(e[1][nm]) for p, e in zip(prev, evs)]))
            prev = [e[1][nm] for e in evs]

    # each preparation alone, calls back to back over copies of its input larger than L2
    # together (X read from HBM every call)
    prep_b2b = {}
    for gname, K, _ in groups:
        n_cp = max(2, -(-int(2.5 * L2_BYTES) // (M * K * 2)))
        xs = [X[gname]] + [X[gname].clone() for _ in range(n_cp - 1)] if M >= 256 else [X[gname]]
        for x in xs:
            sq.prepare(x, cfg, out=A[gname])
        torch.cuda.synchronize()
        n_pc = max(3 * len(xs), 20)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for j in range(n_pc):
            sq.prepare(xs[j % len(xs)], cfg, out=A[gname])
        p1.record(stream)
        torch.cuda.synchronize()
        prep_b2b[gname] = p0.elapsed_time(p1) / n_pc
        del xs

    e2e_value, h2d, d2h = e2e_stack(args, groups, shapes, X, Y, A, QW, WS, cfg, layers, flops,
                                    world, dist, dev)
    value = job_throughput(flops, world, args.steps, ms_max)

    line = None
    if rank == 0:
        hbm, bf16, bf16_sus, peak_src = load_peaks()
        clocks = clk.summary()
        hbm_bound = M < 256  # weight stream dominates below the ridge point (~850 flop/byte)
        has_res = args.residual != "off"
        bpe = prep_bytes_per_elem(args.fmt, args.mask, has_res)
        prep_bytes = sum(M * K * bpe for _, K, _ in groups)
        prep_time = sum(prep_b2b.values())
        gemm_time = sum(gemm_ms.values())
        gemm_tflops = flops / (gemm_time * 1e-3) / 1e12
        method = ((args.fmt, args.mask, args.residual) == ("nvfp4", "pair48", "on")
                  and not args.unfused and M == STACK_M)
        key = f"stack8b_m{M}"
        launches = [{"linear": nm, "M": M, "K": k, "N": n, "ms": gemm_ms[nm],
                     "tflops": lin_flops[nm] / (gemm_ms[nm] * 1e-3) / 1e12,
                     "kernel": gemm_kernel_name(M, n, args.residual)}
                    for nm, (k, n) in shapes.items()]
        if hbm_bound:
            achieved = wbytes / (gemm_time * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "traffic": None,
                    "peak_source": f"{peak_src}: copy bandwidth",
                    "note": "FP4 weight payload (codes and both scale views) of the layer / the "
                            "layer's linear call times (GEMM and split-K sum)",
                    "weight_bytes_per_layer": wbytes, "launches": launches}
        else:
            peak, peak_source = fp4_peak(clocks.get("sm_mhz"), clocks.get("sm_max_mhz"))
            roof = {"bound": "tensor", "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s",
                    "frac": gemm_tflops / peak,
                    "traffic": traffic_from_profile(key) if method else None,
                    "traffic_scope": "DRAM bytes per GEMM launch, mean over the layer's "
                                     f"{len(shapes)} launches",
                    "peak_source": peak_source,
                    "ceiling_frac": metric_ceiling(args.mask, has_res),
                    "executed_frac": gemm_tflops / peak / metric_ceiling(args.mask, has_res),
                    "frac_vs_sustained_peak": gemm_tflops / (bf16_sus * FP4_OVER_BF16),
                    "frac_vs_nominal_peak": gemm_tflops / NOMINAL_FP4_TFLOPS,
                    "note": "2MNK of the layer's linears / the sum of their GEMM launches' "
                            "mean durations (events around each call on the launching stream)",
                    "kernel": gemm_kernel_name(M, 4096, args.residual), "launches": launches}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4",
            "data": "synthetic (drawn on the device: Student-t(4) rows, 0.5 % outlier channels "
                    "x U[20,50] redrawn per row; W ~ N(0, 0.02), random init)",
            "config": {"workload": "stack8b", "M": M, "fused": not args.unfused,
                       "schedule": "pipelined" if args.pipeline else "serial",
                       "launch": (f"CUDA graph of {layers} layers" if args.graph or M < 256
                                  else "eager"),
                       "linears": [f"{nm} {k}x{n}" for nm, (k, n) in shapes.items()],
                       "layers_rotated": layers, "format": args.fmt, "mask": args.mask,
                       "gemm_workspace": {nm: "split-K" if WS[nm] is not None else "none"
                                          for nm in shapes},
                       "residual": args.residual, "out": "bf16",
                       "l2": (f"weights rotate over {layers} layers ({layers * wbytes / 1e6:.0f} MB"
                              f"); X {sum(M * K * 2 for _, K, _ in groups) / 1e6:.0f} MB and Y "
                              f"{sum(M * n * 2 for _, n in shapes.values()) / 1e6:.0f} MB per "
                              "layer" + (" (inputs larger than the 126 MB L2)" if M >= 4096
                                         else "")),
                       "parallelism": f"dp{world}"},
            "roofline": roof,
            "prep": {"ms": prep_time, "gbs": prep_bytes / (prep_time * 1e-3) / 1e9,
                     "hbm_peak_gbs": hbm, "frac": prep_bytes / (prep_time * 1e-3) / 1e9 / hbm,
                     "traffic": prep_traffic_from_profile(key) if method else None,
                     "traffic_scope": "DRAM bytes per preparation call, mean over the layer's "
                                      f"{len(groups)} calls",
                     "bytes_per_elem": bpe, "ms_in_step": sum(prep_ms.values()),
                     "calls": [{"input": gname, "M": M, "K": K, "ms": prep_b2b[gname],
                                "gbs": M * K * bpe / (prep_b2b[gname] * 1e-3) / 1e9}
                               for gname, K, _ in groups],
                     "kernel": " + ".join(prep_kernels(args.fmt, args.mask, args.residual)),
                     "note": "ms: the layer's preparation calls, each timed back to back over "
                             "copies of its input larger than L2 (X from HBM every call); "
                             "ms_in_step: between events around the calls inside the step"},
            "gemm_tflops": gemm_tflops,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": (sum(len(prep_kernels(args.fmt, args.mask, args.residual))
                                 for _ in groups)
                             + sum(1 + (1 if WS[nm] is not None and M < 256 else 0)
                                   for nm in shapes))
                            * args.steps,
            "clocks": clocks,
        }
    # release the layer's buffers before the secondary workload and the CPU baseline
    x_rows, amax_x = {}, {}
    if cpu:
        rows = np.linspace(0, M - 1, min(M, STACK_CPU_ROWS)).astype(np.int64)
        for gname, _, _ in groups:
            xh = X[gname].float().cpu().numpy()
            x_rows[gname] = np.ascontiguousarray(xh[rows])
            amax_x[gname] = S.amax_of(xh)
            del xh
    del X, A, QW, Y, WS
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_secondary and M == STACK_M:
        sub = argparse.Namespace(**vars(args))
        sub.workload, sub.m, sub.steps = "mlp_gate_up", None, min(args.steps, 200)
        sub.no_cpu_baseline, sub.pipeline, sub.given_amax = True, False, False
        d = run_gpu(sub, emit=False, light=True)
        line["secondary"] = [{
            "workload": "mlp_gate_up", "M": 4096, "K": 4096, "N": 14336,
            "value": d["value"], "unit": "TFLOP/s", "steps": sub.steps,
            "gemm_tflops": d["roofline"]["achieved"], "gemm_frac": d["roofline"]["frac"],
            "gemm_traffic": d["roofline"]["traffic"], "prep_gbs": d["prep"]["gbs"],
            "prep_frac": d["prep"]["frac"], "prep_traffic": d["prep"]["traffic"],
            "clocks": d["clocks"]}]
    if cpu:
        samples = stack_cpu_samples(shapes, groups, x_rows, amax_x, w_cols, amax_w,
                                    oracle_modes(args))
        v, passes, t_used, nrows = time_stack_passes(samples, args.cpu_budget, oracle_modes(args))
        line["cpu_baseline"] = {
            "value": v, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{nrows} of {M} rows x {STACK_CPU_COLS} columns of each of the "
                      f"{len(shapes)} linears ({', '.join(shapes)}), {passes} passes, "
                      f"{t_used:.1f} s of CPU work; the weights' sampled columns quantised "
                      "beforehand with each full tensor's amax, the rows prepared with each "
                      "full input's amax"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def e2e_stack(args, groups, shapes, X, Y, A, QW, WS, cfg, layers, flops, world, dist, dev):
    """End to end through the public API with host buffers: every step copies the layer's
    inputs in from pinned memory and its outputs out, on one copy stream per direction that
    overlaps the neighbouring steps' compute (two buffer sets). Returns (TFLOP/s, bytes in,
    bytes out per step)."""
    import torch
    import fp4_sparse_dense_b200 as sq
    n_sets = 2
    stream = torch.cuda.current_stream()
    Xd = [X] + [{k: torch.empty_like(v) for k, v in X.items()} for _ in range(n_sets - 1)]
    Yd = [Y] + [{k: torch.empty_like(v) for k, v in Y.items()} for _ in range(n_sets - 1)]
    xh = [{k: v.cpu().pin_memory() for k, v in X.items()} for _ in range(n_sets)]
    yh = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in Y.items()}
          for _ in range(n_sets)]
    h2d = sum(v.numel() * 2 for v in X.values())
    d2h = sum(v.numel() * 2 for v in Y.values())
    steps = max(1, min(args.steps, 20))
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
    for i in range(steps):
        j = i % n_sets
        with torch.cuda.stream(s_in):
            if i >= n_sets:
                s_in.wait_event(ev_done[j])  # step i - n_sets has read these inputs
            for k in Xd[j]:
                Xd[j][k].copy_(xh[j][k], non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= n_sets:
            stream.wait_event(ev_out[j])  # the outputs of step i - n_sets have been copied out
        lw = QW[i % layers]
        for gname, _, names in groups:
            a = sq.prepare(Xd[j][gname], cfg, out=A[gname])
            for nm in names:
                sq.linear(a, lw[nm], out=Yd[j][nm], workspace=WS[nm])
        ev_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            for k in Yd[j]:
                yh[j][k].copy_(Yd[j][k], non_blocking=True)
            ev_out[j].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    value = job_throughput(flops, world, steps, max_over_ranks(e0.elapsed_time(e1), dist, dev))
    assert sq.sharq_device_status() == 0
    return value, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sharq", choices=["sharq", "reference"])
    ap.add_argument("--workload", default="stack8b", choices=["stack8b"] + list(WORKLOADS),
                    help="stack8b: the 8B-shaped layer (default, M = 8192); the others are "
                         "single linears")
    ap.add_argument("--m", type=int, default=None,
                    help=f"token rows: of --workload stack8b (default {STACK_M}), or replacing "
                         "a single-linear workload's M (decode sizes)")
    ap.add_argument("--unfused", action="store_true",
                    help="stack8b: the seven linears as separate GEMMs (default: q|k|v and "
                         "gate|up weights concatenated along N, four GEMMs per layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="stack8b at the default M: skip the mlp_gate_up figures added to the line")
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
        if args.given_amax or args.mask == "pair48_given":
            raise SystemExit("stack8b runs the method's preparation (no --given-amax, no "
                             "supplied mask)")
        return run_stack(args)
    run_gpu(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
