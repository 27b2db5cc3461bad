"""bench.py keeps its one-line JSON contract: a short run on the GPU prints exactly one JSON
line with the keys the measurement needs (metric and value, the roofline of the dominant
kernel with its traffic, the preparation's figures, the end-to-end number with the bytes
it copies, the launch count and the clock record)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "4",
                          "--warmup", "3", "--no-cpu-baseline", *args],
                         capture_output=True, text=True, cwd=ROOT, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def _contract_keys(d):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "prep", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]


def test_default_line_is_the_8b_layer_at_8192_rows():
    """The default run measures the 8B-shaped layer (fused q|k|v and gate|up) at M = 8192,
    the largest prefill of the sweep, with the GEMM fraction against 4 x the bf16 burst peak,
    the host-buffer e2e number, and mlp_gate_up as a secondary figure."""
    d = _run()
    _contract_keys(d)
    assert d["steps"] == 4 and d["warmup"] == 3 and d["n_gpus"] == 1
    c = d["config"]
    assert c["workload"] == "stack8b" and c["M"] == 8192 and c["fused"] is True
    r = d["roofline"]
    assert r["bound"] == "tensor" and "burst" in r["peak_source"]
    assert len(r["launches"]) == 4
    flops = sum(2.0 * 8192 * k * n for k, n in [(4096, 6144), (4096, 4096), (4096, 28672),
                                                 (14336, 4096)])
    assert abs(d["value"] - flops / (d["ms_per_step"] * 1e-3) / 1e12) < 1e-6 * d["value"]
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 8192 * (3 * 4096 + 14336) * 2
    assert e["d2h_bytes_per_step"] == 8192 * (6144 + 4096 + 28672 + 4096) * 2
    assert d["gpu_launches"] == (4 * 2 + 4) * 4  # two preparation kernels per input, 4 GEMMs
    assert len(d["prep"]["calls"]) == 4 and d["prep"]["gbs"] > 0
    sec = d["secondary"][0]
    assert sec["workload"] == "mlp_gate_up" and sec["gemm_tflops"] > 0


def test_single_linear_line_has_the_contract_keys():
    d = _run("--workload", "mlp_gate_up")
    _contract_keys(d)
    assert d["config"]["workload"] == "mlp_gate_up" and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and "burst" in r["peak_source"]
    assert r["traffic"] is not None  # the committed capture matches the current GEMM code
    assert d["prep"]["issue_roofline"] is not None
    assert d["prep"]["traffic"] is not None
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 4096 * 4096 * 2 and e["d2h_bytes_per_step"] == 4096 * 14336 * 2
    assert d["gpu_launches"] == 3 * 4  # mask, quantisation and GEMM per step


def test_bench_given_amax_mode():
    d = _run("--workload", "mlp_gate_up", "--given-amax")
    assert d["prep"]["kernel"] == "prep_pair_kernel"
    assert d["gpu_launches"] == 2 * 4
    assert d["roofline"]["traffic"] is None  # the capture is of the default mode only


def test_bench_decode_rows():
    """--m replaces a single-linear workload's token rows: below 256 rows the line's roofline
    is the weight stream against HBM, the weights rotate over copies larger than L2, and
    the split-K summing kernel is counted among the launches."""
    d = _run("--workload", "mlp_down", "--m", "1")
    assert d["config"]["M"] == 1 and d["config"]["workload"] == "mlp_down"
    assert "CUDA graph" in d["config"]["launch"]  # device time, not host launch latency
    assert "copies" in d["config"]["l2"]
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["split_k"] is True
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["gpu_launches"] == 4 * 4  # mask, quantisation, GEMM, split-K sum per step
