"""Failure detection on the GPU without a fault: every pipeline wait in the
kernels is bounded, and an expired wait is reported through the device status
word.  fa2_watchdog_selftest makes one such wait run out (an mbarrier that no
thread arrives on, limit of a few milliseconds); the test checks the status
the host reads, that clearing it works, and that the context still computes
correct attention afterwards.  Nothing here traps, faults or spins without a
limit.  (The file name sorts it after the parity tests.)"""
import time

import numpy as np
import pytest
import torch

import fa2_inputs
from parity_util import assert_close, default_scale, gpu_fwd_bwd, to64

pytestmark = pytest.mark.gpu

FA2_OK = 0
FA2_ERR_DEVICE_TIMEOUT = 8


def test_expired_wait_is_reported_and_context_survives(oracle_mod):
    import causal_attention_fa2_b200 as fa2
    torch.cuda.synchronize()
    fa2.clear_device_status()
    assert fa2.last_device_status() == FA2_OK

    t0 = time.perf_counter()
    fa2.watchdog_selftest(limit_ns=2_000_000)          # 2 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert fa2.last_device_status() == FA2_ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0, f"the bounded wait took {elapsed:.3f} s"

    # A second expiry keeps the first recorded error; clearing resets it.
    fa2.watchdog_selftest(limit_ns=1_000_000)
    torch.cuda.synchronize()
    assert fa2.last_device_status() == FA2_ERR_DEVICE_TIMEOUT
    fa2.clear_device_status()
    assert fa2.last_device_status() == FA2_OK

    # The context is still usable: a small causal forward + backward matches
    # the fp64 oracle and records no error.
    B, H, N, d = 1, 2, 200, 64
    inp = fa2_inputs.make_inputs(B, H, N, d, "bf16", seed=17)
    scale = default_scale(d)
    got = gpu_fwd_bwd(inp, True, scale)
    q, k, v, do = (to64(inp[n]) for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = oracle_mod.forward(q, k, v, True, scale)
    dq_ref, dk_ref, dv_ref = oracle_mod.backward(q, k, v, do, True, scale)
    for name, ref in (("o", o_ref), ("lse", lse_ref), ("dq", dq_ref), ("dk", dk_ref), ("dv", dv_ref)):
        assert_close(to64(got[name]), np.asarray(ref), "bf16", name)
    assert fa2.last_device_status() == FA2_OK


def test_selftest_rejects_out_of_range_limits():
    import causal_attention_fa2_b200 as fa2
    for bad in (0, 999, 10**10 + 1):
        with pytest.raises(fa2.FA2Error):
            fa2.watchdog_selftest(limit_ns=bad)
