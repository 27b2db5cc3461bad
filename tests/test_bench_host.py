"""Host-side helpers of bench.py on CPU: the --m override of a workload's token rows, the
inputs drawn for it, and the oracle's CPU baseline counting only the rows it really ran."""
import argparse

import pytest


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
