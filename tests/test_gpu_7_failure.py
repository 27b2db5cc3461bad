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
