"""The device-side watchdog, tested without faulting, trapping or hanging the
GPU: a bounded wait on a barrier that nothing completes must give up after its
time limit, report FA_ERR_DEVICE_TIMEOUT through the status word, and leave the
context usable for the next forward."""
import time

import numpy as np
import pytest

from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, run_gpu

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    assert fa.fa_get_device_status() == fa.FA_OK
    t0 = time.time()
    assert fa.fa_selftest_watchdog(100) == fa.FA_OK
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert 0.09 <= elapsed < 5.0, elapsed
    assert fa.fa_get_device_status() == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_get_device_status() == fa.FA_OK          # read and cleared
    # the context still computes correct results
    w = syn.config("c1").draw()
    o, lse, st = run_gpu(w)
    assert st == fa.FA_OK
    import oracle
    assert_parity(o, lse, *oracle.attention(w.q, w.k, w.v, 1, 1, 1, 256, 64, w.scale, False), "after watchdog")


def test_selftest_rejects_out_of_range_timeouts():
    from exact_tiled_attention_32_b200 import binding as fa
    assert fa.fa_selftest_watchdog(0) == fa.FA_ERR_SHAPE
    assert fa.fa_selftest_watchdog(5000) == fa.FA_ERR_SHAPE
