"""Failure detection on the GPU without a fault: the fused kernel's bounded
waits.

ssd_selftest_timeout launches the fused tensor-core kernel with its TMA loads
withheld, so every wait on them runs out after about a second; the kernel
records the timeout in the device status word, drains and exits.  The host
reads SSD_ERR_TIMEOUT through ssd_read_device_status, and the same context
then runs a normal scan that still matches the oracle.
"""
import time

import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu

SSD_OK = 0
SSD_ERR_TIMEOUT = 8


@pytest.mark.parametrize("two_heads", [False, True])
def test_withheld_loads_time_out_and_context_survives(two_heads):
    """Both fused kernels: the one-head one (default) and the two-head one."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl = inputs.custom("mamba2_130m_layer", batch=1, seqlen=512, nheads=2)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    assert ssd.ssd_read_device_status() == SSD_OK  # nothing pending before

    t0 = time.monotonic()
    ssd.ssd_selftest_timeout(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                             chunk=wl.chunk, two_heads=two_heads)
    status = ssd.ssd_read_device_status()  # synchronises the stream
    elapsed = time.monotonic() - t0
    assert status == SSD_ERR_TIMEOUT
    assert elapsed < 30.0, elapsed  # bounded: about one second per wait chain
    assert ssd.ssd_read_device_status() == SSD_OK  # reading cleared the word

    # the context is intact: a normal scan right after matches the oracle
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, two_heads=two_heads)
    torch.cuda.synchronize()
    assert ssd.ssd_read_device_status() == SSD_OK
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]


@pytest.mark.parametrize("two_heads", [True])
def test_carry_wait_times_out_and_context_survives(two_heads):
    """The two-head kernel's segmented schedule with no carry ever published:
    every segment after the first gives up waiting for its predecessor's state
    after about two seconds; the host reads SSD_ERR_TIMEOUT, and a normal scan
    (with its carries) then matches the oracle in the same context."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=300, nheads=160, ngroups=1, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    assert ssd.ssd_read_device_status() == SSD_OK
    ssd.ssd_selftest_set_segments(3)
    try:
        t0 = time.monotonic()
        ssd.ssd_selftest_carry_timeout(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                       chunk=wl.chunk, two_heads=two_heads)
        status = ssd.ssd_read_device_status()
        elapsed = time.monotonic() - t0
        assert status == SSD_ERR_TIMEOUT
        assert elapsed < 30.0, elapsed
        assert ssd.ssd_read_device_status() == SSD_OK
        y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                  chunk=wl.chunk, two_heads=two_heads)
        torch.cuda.synchronize()
    finally:
        ssd.ssd_selftest_set_segments(0)
    assert ssd.ssd_read_device_status() == SSD_OK
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
