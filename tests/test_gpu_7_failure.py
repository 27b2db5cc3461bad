"""Failure detection on the GPU without a fault: a bounded wait on a flag that nothing sets
runs out, the kernel records SHARQ_ERR_TIMEOUT and returns, sharq_device_status reports it
once (and clears it), and the context stays usable for the hot path."""
import ctypes
import time

import numpy as np
import pytest

from oracle import sharq as S
from tests.gpu_helpers import act_bytes, assert_bytes_equal, to_device
from workloads import heavy_activations

pytestmark = pytest.mark.gpu


def _probe(sq, flag, expected, limit_ns):
    import torch
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sq.sharq_wait_probe(ctypes.c_void_p(flag.data_ptr()), expected, limit_ns, stream)
    assert rc == 0, sq.sharq_status_string(rc)


def test_bounded_wait_reports_timeout_and_context_survives():
    import fp4_sparse_dense_b200 as sq
    import torch
    assert sq.sharq_device_status() == 0
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")  # nothing ever sets it
    t0 = time.perf_counter()
    _probe(sq, flag, 1, 50_000_000)  # 50 ms
    assert sq.sharq_device_status() == 5  # SHARQ_ERR_TIMEOUT, read after the wait ran out
    assert time.perf_counter() - t0 >= 0.045
    assert sq.sharq_device_status() == 0  # reported once
    # the context still runs the hot path correctly
    x = heavy_activations(np.random.default_rng(1), 64, 512)
    act = sq.prepare(to_device(x), sq.Config())
    torch.cuda.synchronize()
    assert sq.sharq_device_status() == 0
    assert_bytes_equal(act_bytes(act), S.act_buffers(S.prepare(x.values)))


def test_wait_that_is_satisfied_reports_nothing():
    import fp4_sparse_dense_b200 as sq
    import torch
    flag = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    _probe(sq, flag, 7, 5_000_000_000)
    assert sq.sharq_device_status() == 0
    assert time.perf_counter() - t0 < 1.0


def test_timeout_is_reported_on_its_own_stream_once():
    """A probe that times out on stream A while stream B runs the preparation: reading B's
    status syncs only B and reports nothing (A is still waiting), reading A's reports the
    timeout once, and the device-wide read afterwards finds nothing left."""
    import fp4_sparse_dense_b200 as sq
    import torch
    assert sq.sharq_device_status() == 0
    x = heavy_activations(np.random.default_rng(2), 256, 1024)
    xd = to_device(x)
    cfg = sq.Config()
    sq.prepare(xd, cfg)  # warm: the kernels are loaded before the timed part
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")  # nothing ever sets it
    t0 = time.perf_counter()
    rc = sq.sharq_wait_probe(ctypes.c_void_p(flag.data_ptr()), 1, 400_000_000,
                             ctypes.c_void_p(sa.cuda_stream))  # 400 ms on stream A
    assert rc == 0
    with torch.cuda.stream(sb):
        act = sq.prepare(xd, cfg, stream=sb)
    assert sq.sharq_read_device_status(ctypes.c_void_p(sb.cuda_stream)) == 0
    t_b = time.perf_counter() - t0
    assert t_b < 0.3, t_b  # B's read did not wait for A's probe
    assert sq.sharq_read_device_status(ctypes.c_void_p(sa.cuda_stream)) == 5  # TIMEOUT
    assert time.perf_counter() - t0 >= 0.35
    assert sq.sharq_read_device_status(ctypes.c_void_p(sa.cuda_stream)) == 0  # reported once
    assert sq.sharq_device_status() == 0
    assert_bytes_equal(act_bytes(act), S.act_buffers(S.prepare(x.values)))
