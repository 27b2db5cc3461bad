"""Host-side helpers of bench.py on CPU: the --m override of a workload's token rows, the
inputs drawn for it, the oracle's CPU baseline counting only the rows it really ran, the
roofline's algorithmic bytes and ceilings, the clock-aware peak, and the gating of the
committed ncu records by the source they were taken on."""
import argparse
import json
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture
def bench(monkeypatch):
    import bench as b
    monkeypatch.setitem(b.WORKLOADS, "tiny_linear", (32, 256, 128, True))
    return b


def _args(workload, m=None):
    return argparse.Namespace(workload=workload, m=m)


def test_workload_shape_and_row_override(bench):
    assert bench.workload_shape(_args("mlp_gate_up")) == (4096, 4096, 14336)
    assert bench.workload_shape(_args("mlp_down", 8)) == (8, 14336, 4096)
    assert bench.workload_shape(_args("tiny_linear", 3)) == (3, 256, 128)


def test_inputs_follow_the_row_override(bench):
    x, w = bench.make_inputs("tiny_linear", 7, 3)
    assert x.values.shape == (3, 256) and w.values.shape == (256, 128)
    x32, _ = bench.make_inputs("tiny_linear", 7)
    assert x32.values.shape == (32, 256)


@pytest.mark.parametrize("M", [1, 20])
def test_cpu_baseline_counts_the_rows_it_ran(bench, M):
    from oracle import sharq as S
    x, w = bench.make_inputs("tiny_linear", 3, M)
    qw = S.quantize_weight(w.values)
    value, cores, sample = bench.cpu_baseline("tiny_linear", 30.0, x, qw,
                                              {"fmt": "nvfp4", "mask": "pair48",
                                               "residual": True})
    assert sample.startswith(f"{M} of {M} rows")  # every row once, none counted twice
    assert value > 0 and cores >= 1


def test_input_sets_exceed_l2(bench):
    for M, K, N in [(4096, 4096, 14336), (2048, 4096, 4096), (4096, 14336, 4096), (256, 4096, 4096)]:
        n = bench.input_sets(M, K, N)
        assert n >= 3 and n * (M * K + M * N) * 2 >= 2.5 * bench.L2_BYTES
    assert bench.input_sets(4096, 4096, 14336) == 3  # the default workload is unchanged
    assert bench.input_sets(1, 14336, 4096) == 3     # decode rotates its weights instead


def test_stack_layout_covers_the_seven_linears(bench):
    fused, fgroups = bench.stack_layout(False)
    unfused, ugroups = bench.stack_layout(True)
    flops = lambda sh: sum(k * n for k, n in sh.values())  # noqa: E731
    assert flops(fused) == flops(unfused)  # concatenation along N keeps the work
    assert set(fused) == {"qkv", "o", "gate_up", "down"} and len(unfused) == 7
    for shapes, groups in ((fused, fgroups), (unfused, ugroups)):
        names = [nm for _, _, nms in groups for nm in nms]
        assert sorted(names) == sorted(shapes)
        for _, K, nms in groups:
            assert all(shapes[nm][0] == K for nm in nms)


def test_stack_cpu_sample_counts_what_it_ran(bench):
    """The reference arm's layer sample: whole passes over every linear, FLOPs counted from
    the rows and columns actually multiplied."""
    args = argparse.Namespace(unfused=False, fmt="nvfp4", mask="pair48", residual="on")
    samples = bench.reference_stack_samples(args, 11)
    assert [s["name"] for s in samples] == ["qkv", "o", "gate_up", "down"]
    for s in samples:
        assert s["x"].shape == (bench.STACK_CPU_ROWS, s["K"])
        assert s["qw"].wq.shape == (bench.STACK_CPU_COLS, s["K"])
    v, passes, t, rows = bench.time_stack_passes(samples, 0.0, bench.oracle_modes(args))
    assert passes == 1 and rows == bench.STACK_CPU_ROWS and v > 0
    flops = sum(2.0 * rows * bench.STACK_CPU_COLS * s["K"] for s in samples)
    assert abs(v - flops / t / 1e12) < 1e-9


def test_reference_arm_reports_the_time_it_ran(bench, capsys, monkeypatch):
    """ms_per_step is the real duration of a sample step, so steps x ms_per_step is the
    CPU time the arm spent (not an extrapolation to a full-size step)."""
    import json
    import time
    monkeypatch.setenv("RANK", "0")
    args = argparse.Namespace(workload="stack8b", m=None, unfused=False, fmt="nvfp4",
                              mask="pair48", residual="on", steps=2, warmup=1, gpus=1)
    t0 = time.perf_counter()
    assert bench.run_reference(args) == 0
    wall = time.perf_counter() - t0
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["steps"] == 2
    assert d["steps"] * d["ms_per_step"] * 1e-3 <= wall
    assert d["config"]["workload"] == "stack8b" and d["config"]["M"] == 8192


def test_fp4_peak_follows_the_clock_of_the_timed_region(monkeypatch):
    """A burst at full clock is held to 4 x the bf16 burst figure; a run under the power cap
    (median below 90 % of the maximum clock) to 4 x the sustained figure scaled to its clock."""
    import bench
    monkeypatch.setattr(bench, "load_peaks", lambda: (6541.5, 1654.2, 1383.4, "measured"))
    monkeypatch.setattr(bench, "sustained_clock_mhz", lambda: 1327.0)
    p, src = bench.fp4_peak(1965.0, 1965.0)
    assert p == pytest.approx(4 * 1654.2) and "burst" in src
    p, src = bench.fp4_peak(1800.0, 1965.0)          # within 10 % of max: still a burst
    assert p == pytest.approx(4 * 1654.2)
    p, src = bench.fp4_peak(1515.0, 1965.0)
    assert p == pytest.approx(4 * 1383.4 * 1515.0 / 1327.0) and "sustained" in src
    p, src = bench.fp4_peak(None, None)              # no clock samples: the burst figure
    assert p == pytest.approx(4 * 1654.2)
    monkeypatch.setattr(bench, "sustained_clock_mhz", lambda: None)
    assert bench.fp4_peak(1515.0, 1965.0)[0] == pytest.approx(4 * 1654.2)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("mask", ["pair48", "elem24", "none"])
@pytest.mark.parametrize("residual", [True, False])
def test_prep_bytes_per_elem_is_the_output_layout(fmt, mask, residual):
    """The preparation roofline's algorithmic bytes per element = the 16-bit read plus every
    byte of the oracle's output buffers (a shape without tile padding: 128 rows, K / block a
    multiple of 4)."""
    import bench
    from oracle import sharq as S
    M, K = 128, 512
    x = np.random.default_rng(1).standard_normal((M, K)).astype(np.float32)
    bufs = S.act_buffers(S.prepare(x, fmt, mask, residual=residual))
    out = sum(v.size for k, v in bufs.items() if k != "tensor_scale" and v is not None)
    assert bench.prep_bytes_per_elem(fmt, mask, residual) == pytest.approx(2.0 + out / (M * K))


def test_metric_ceiling_from_the_mma_rates():
    """2MNK / t at full tensor-pipe use over the dense FP4 peak: the sparse backbone runs at
    twice the dense rate, a dense residual adds its own pass."""
    import bench
    assert bench.metric_ceiling("pair48", True) == pytest.approx(2 / 3)
    assert bench.metric_ceiling("pair48", False) == pytest.approx(2.0)
    assert bench.metric_ceiling("elem24", True) == pytest.approx(0.5)
    assert bench.metric_ceiling("none", False) == pytest.approx(1.0)


def test_gemm_kernel_choice():
    import bench
    assert bench.gemm_kernel_name(256, 4096) == "sharq_gemm_pair_kernel"
    assert bench.gemm_kernel_name(8192, 28672) == "sharq_gemm_pair_kernel"
    assert bench.gemm_kernel_name(255, 4096) == "sharq_gemm_kernel"     # decode-sized rows
    assert bench.gemm_kernel_name(4096, 384) == "sharq_gemm_kernel"     # N not a multiple of 256
    assert bench.gemm_kernel_name(4096, 4096, "own") == "sharq_gemm_kernel"  # two accumulators


def test_traffic_records_follow_the_code_not_the_comments(tmp_path, monkeypatch):
    """A committed ncu record is reported only while it matches the hash of the GEMM sources;
    comment and spacing edits keep the hash, a code edit drops the record."""
    import shutil
    import bench
    for f in bench.GEMM_SRC:
        (tmp_path / f).parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, f), tmp_path / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"mlp_gate_up": {"dram_bytes_per_launch": 123, "gemm_src": bench.src_hash(bench.GEMM_SRC)}}
    (tmp_path / "profiles" / "gemm_traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_from_profile("mlp_gate_up") == 123
    assert bench.traffic_from_profile("attn_proj") is None           # no record for it
    src = tmp_path / bench.GEMM_SRC[0]
    src.write_text(src.read_text() + "\n// a note\n/* and another */\n\n")
    assert bench.traffic_from_profile("mlp_gate_up") == 123           # comments only
    src.write_text(src.read_text() + "\nstatic int sharq_extra_symbol = 1;\n")
    assert bench.traffic_from_profile("mlp_gate_up") is None          # the code changed
