"""Failure detection without a GPU fault: every device wait of the library is
bounded and, when its limit passes, records KL_ERR_DEVICE_TIMEOUT in the
per-device status word and returns.  kl_selftest_wait_timeout runs that same
wait on an mbarrier nothing ever arrives on (no copy, MMA or TMEM in flight),
with a 1 ms limit, so the timeout path is taken for real; the host then reads
the status, clears it, and the context keeps working."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import nvfp4
from synth import normal_bf16

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports_it():
    assert kl.device_status(clear=True) in ("KL_OK", "KL_ERR_DEVICE_TIMEOUT", "KL_ERR_NONFINITE")
    assert kl.device_status() == "KL_OK"
    waited = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    kl.selftest_wait_timeout(1_000_000, waited)   # 1 ms
    stop.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop)
    assert 1.0 <= ms < 200.0, ms                  # it waited its limit, then returned
    assert int(waited.item()) == 0                # the wait gave up
    assert kl.device_status(clear=False) == "KL_ERR_DEVICE_TIMEOUT"
    assert kl.device_status(clear=True) == "KL_ERR_DEVICE_TIMEOUT"
    assert kl.device_status() == "KL_OK"          # cleared


def test_context_stays_usable_after_a_timeout():
    kl.selftest_wait_timeout(1_000_000)
    assert kl.device_status(clear=True) == "KL_ERR_DEVICE_TIMEOUT"
    x = normal_bf16((256, 512), 3)
    q = kl.quantize_nvfp4(x.cuda(), layout="linear")
    torch.cuda.synchronize()
    codes, scales, gs = nvfp4.quantize(x.float().numpy())
    np.testing.assert_array_equal(q.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(q.scales.cpu().numpy(), scales)
    assert kl.device_status() == "KL_OK"
