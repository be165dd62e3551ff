"""Failure detection of the device-side bounded waits, without a GPU fault: a
self-test kernel waits on an mbarrier that nothing completes, gives up after a
short cycle limit and records the timeout the way every kernel wait does; the
host reads it through bq_device_status and the context keeps working."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_quant_b200 as bq
from _helpers import Problem, reference, assert_within_tolerance

BQ_ERR_SHAPE, BQ_ERR_TIMEOUT = 2, 6


def test_selftest_rejects_bad_limits():
    L = bq.lib()
    assert L.bq_selftest_wait_timeout(10, None) == BQ_ERR_SHAPE
    assert L.bq_selftest_wait_timeout(5_000_000_000, None) == BQ_ERR_SHAPE


@pytest.mark.gpu
def test_timed_out_wait_is_reported_and_context_survives():
    L = bq.lib()
    assert L.bq_device_status() == 0                       # clean start
    assert L.bq_selftest_wait_timeout(2_000_000, None) == 0   # ~1 ms of SM clocks
    assert L.bq_device_status() == BQ_ERR_TIMEOUT          # reported ...
    assert L.bq_device_status() == 0                       # ... and cleared
    # the context still runs kernels correctly
    p = Problem("q4_0", 256, 512, seed=3)
    wq, s, _ = p.device()
    x = p.x(40)
    y = bq.quant_matmul(x.cuda(), wq, s, None, 32, 4)
    torch.cuda.synchronize()
    y_ref, a_ref = reference(x, p.wb)
    assert_within_tolerance(y, y_ref, a_ref, "after a timed-out wait")
    assert L.bq_device_status() == 0
