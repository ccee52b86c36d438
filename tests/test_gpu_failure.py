"""Failure detection on the GPU without a fault: a bounded wait runs out.

The tensor-core kernels bound every mbarrier wait; when one gives up it
records SWAT_ERR_TIMEOUT in the device status word and returns. Here the
library's check kernel waits on a barrier phase that nothing completes, with
a short limit; the test reads the status and then runs attention on the same
context to show that it is still usable.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
from sliding_window_sigmoid_b200 import binding, inputs
from tests.helpers import assert_bf16_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    assert binding.device_status() == 0
    t0 = time.perf_counter()
    binding.check_wait_timeout(50_000_000)          # 50 ms of device time
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert binding.device_status() == -4            # SWAT_ERR_TIMEOUT, read and cleared
    assert binding.device_status() == 0
    assert 0.04 < elapsed < 5.0
    # the same context still computes
    q, k, v = inputs.qkv(1, 200, 2, 2, 64, seed=3, scale=0.125, dtype=torch.bfloat16)
    sl = inputs.balanced_alibi_slopes(2)
    o, _ = binding.attn_fwd(q.cuda(), k.cuda(), v.cuda(), window=64, slopes=sl, rope_base=1e4)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    ref, _ = oracle.swat_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), window=64,
                             slopes=sl.numpy(), rope_base=1e4)
    assert_bf16_close(o, ref, "after timeout")
