"""Failure detection of the device-side waits, without faulting or hanging a GPU.

Every wait in the prefill kernel (ring flags in global memory, mbarriers in
shared memory) is bounded: when it runs out it sets the library's device
error word and the kernel returns. gdn_wait_selftest runs both kinds of wait
on objects nothing ever signals, with a short limit; gdn_device_error must
then report GDN_ERR_DEVICE_TIMEOUT once, clear the word, and the context must
still compute correct results.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

gdn = pytest.importorskip("gated_deltanet_linear_21_b200")


def test_wait_selftest_rejects_out_of_range_limits():
    lib = gdn.lib()
    for bad in (0, -5, 1000001):
        assert lib.gdn_wait_selftest(bad, None) == gdn.GDN_ERR_INVALID_ARG
        assert "max_wait_us" in lib.gdn_last_error().decode()


@pytest.mark.gpu
def test_bounded_waits_time_out_and_the_context_survives():
    gdn.device_error()                       # start from a clear error word
    gdn.wait_selftest(2000)
    with pytest.raises(gdn.GdnError) as err:
        gdn.device_error()
    assert err.value.status == gdn.GDN_ERR_DEVICE_TIMEOUT
    gdn.device_error()                       # reported once, then cleared
    # the context still computes: one decode step against the oracle
    B, Hqk, Hv, d = 2, 2, 4, 128
    state = workloads.decode_state(B, Hv, d, std=0.05)
    ref_state = state.double().numpy().copy()
    x = workloads.decode_step_inputs(0, B, Hqk, Hv, d)
    sd = state.cuda()
    o = gdn.decode(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["g"].cuda(), x["beta"].cuda(), sd)
    ro, ref_state = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], ref_state)
    assert np.abs(o.float().cpu().double().numpy() - ro).max() <= 2e-2
    assert np.abs(sd.cpu().double().numpy() - ref_state).max() <= 1e-2
    gdn.device_error()
