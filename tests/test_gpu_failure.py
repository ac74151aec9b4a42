"""The bounded-wait failure path, exercised without a fault: a wait on a barrier
that nothing completes gives up, the device status word reads HD_ERR_TIMEOUT,
the tensor-core kernels skip their work while it is recorded, and after it is
cleared the same call computes the right result on the same context."""
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import O_MAX, O_MEAN, check, host64, need_gpu

pytestmark = pytest.mark.gpu


def test_timeout_is_recorded_and_kernels_skip_until_cleared():
    need_gpu()
    assert hd.hd_device_status(clear=True) == hd.HD_OK
    hd.hd_selftest_wait_timeout(2_000_000)  # ~1 ms of SM clock
    assert hd.hd_device_status(clear=False) == hd.HD_ERR_TIMEOUT

    inp = syn.attention_inputs(1, 40, 2, 2, 1, 64, seed=3)
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    out = torch.full_like(q, 7.0)
    lse = torch.full((1, 2, 80), 7.0, dtype=torch.float32, device="cuda")
    hd.hd_attn_fwd(q, k, v, out, lse, 1, 40, 2, 2, 1, 64, hd.CROSS_FULL, 0, 0, 0.125)
    torch.cuda.synchronize()
    # the recorded timeout makes the kernel return before any work
    assert (out == 7.0).all() and (lse == 7.0).all()
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_TIMEOUT

    assert hd.hd_device_status(clear=True) == hd.HD_OK
    hd.hd_attn_fwd(q, k, v, out, lse, 1, 40, 2, 2, 1, 64, hd.CROSS_FULL, 0, 0, 0.125)
    torch.cuda.synchronize()
    assert hd.hd_device_status() == hd.HD_OK
    o_ref, _ = oracle.attn_fwd(inp["q"], inp["k"], inp["v"], 2, hd.CROSS_FULL, 1, False, 0.125)
    check(host64(out), o_ref, O_MAX, O_MEAN, "O after clearing")


def test_timeout_limit_is_honoured_quickly():
    """A short limit ends the wait in about that time, not the kernels' ~2 s."""
    need_gpu()
    hd.hd_device_status(clear=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hd.hd_selftest_wait_timeout(20_000_000)  # ~10 ms at ~2 GHz
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert 1.0 < ms < 500.0, ms
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_TIMEOUT
