"""Multi-process host logic of the benchmark on CPU (gloo, world size 2): every rank draws
its own batch, the timing reduction takes the slowest rank, and the job throughput counts
all ranks' work. No GPU and no collective on the data path."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = [12.0, 30.0][rank]
    ms_max = bench.max_over_ranks(ms, dist, "cpu")
    value = bench.job_throughput(2e12, world, 10, ms_max)
    q.put((rank, bench.rank_seed(rank), ms_max, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    (r0, s0, m0, v0), (r1, s1, m1, v1) = res
    assert s0 != s1                      # independent batches per rank
    assert m0 == m1 == 30.0              # slowest rank's time on every rank
    assert v0 == v1 == pytest.approx(2e12 * 2 * 10 / 0.030 / 1e12)


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(5.0, None, "cpu") == 5.0
    assert bench.job_throughput(1e12, 1, 1, 1000.0) == pytest.approx(1.0)


def _ref_worker(rank, world, q):
    import argparse
    import contextlib
    import io
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    args = argparse.Namespace(workload="stack8b", m=None, unfused=False, fmt="nvfp4",
                              mask="pair48", residual="on", steps=1, warmup=1, gpus=world)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.run_reference(args)
    q.put((rank, rc, out.getvalue()))


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm (the CPU oracle) runs and prints on rank 0 only; the
    other ranks exit 0 without work or output."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ref_worker, args=(r, 2, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = dict((r, (rc, txt)) for r, rc, txt in (q.get(timeout=5) for _ in range(2)))
    assert res[1] == (0, "")
    rc0, txt0 = res[0]
    lines = [ln for ln in txt0.splitlines() if ln.startswith("{")]
    assert rc0 == 0 and len(lines) == 1 and '"impl": "reference"' in lines[0]
