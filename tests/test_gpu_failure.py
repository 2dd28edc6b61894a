"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The self-test kernel waits, through the library's bounded mbarrier wait, on a
barrier that nothing completes. The wait must give up after its limit, the
timeout must reach the host through the status word, and the context must stay
usable: a layer run right after it still matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import block_sparse_linear_sm_b200 as sla
from block_sparse_linear_sm_b200 import workloads as wl

from gpu_util import DeviceRun, full_errors

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_is_reported():
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    sla.sla_selftest_wait_timeout(ws, 2_000_000)  # 2 ms
    st, detail = sla.sla_check_device_status(ws)
    elapsed = time.time() - t0
    assert (st, detail) == (sla.SLA_ERR_DEVICE_TIMEOUT, 300)
    assert elapsed < 5.0
    # the status word was cleared by the check
    assert sla.sla_check_device_status(ws) == (sla.SLA_OK, 0)


def test_context_usable_after_a_timeout():
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    sla.sla_selftest_wait_timeout(ws, 1_000_000)
    assert sla.sla_check_device_status(ws)[0] == sla.SLA_ERR_DEVICE_TIMEOUT
    cfg = wl.small_config(name="after_timeout", N=1024, N_valid=1000, d=128, k_h=3, k_l=4)
    run = DeviceRun(cfg)
    err = full_errors(run, run.layer().forward())
    assert err["max_abs"] <= 2e-2 and err["mean_abs"] <= 2e-3, err
