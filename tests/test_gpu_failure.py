"""Failure detection without a GPU fault: every pipeline wait in the kernels
is bounded and, when it gives up, records a bit in the library's device
error word and lets the kernel return. Here a wait is made to run out (an
mbarrier that nothing arrives on, with a 20 ms limit); the host reads the
status, and the same context then runs a GEMV that matches the oracle."""
import numpy as np
import pytest
import torch

import ternary_absmax_int8_b200 as tq
from tests._gpu import assert_parity, gpu_forward, host_pack, oracle_forward
from workloads import make_projections

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives(cuda_device):
    assert tq.tq_device_error(reset=True) == 0
    tq.tq_selftest_wait_timeout(20_000)
    torch.cuda.synchronize()
    assert tq.tq_device_error(reset=True) == 1     # kErrWaitTimeout
    assert tq.tq_device_error(reset=False) == 0    # cleared
    p = next(make_projections([("q_proj", 2560, 2560)], M=1, seed=12))
    assert_parity(gpu_forward(host_pack(p.w), p.N, p.w_scale, p.x_bf16),
                  oracle_forward(p.w, p.w_scale, p.x_bf16), "after the timeout")
    assert tq.tq_device_error(reset=True) == 0


def test_selftest_rejects_unbounded_limits(cuda_device):
    for bad in (0, 2_000_001):
        with pytest.raises(tq.TQError) as e:
            tq.tq_selftest_wait_timeout(bad)
        assert e.value.name == "TQ_ERR_VALUE"
