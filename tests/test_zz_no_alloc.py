"""ssd_scan_fwd_noalloc: the step-by-step scan for callers that cannot
allocate device memory (graph capture in progress, engines that plan memory
up front, fixed-budget runtimes).  Its scratch is a buffer compiled into
libssd.so instead of a caller workspace.

The tests call it through the C ABI twice in a row, on different inputs, and
compare each result with ssd_scan_fwd_unfused (same kernels, caller
workspace) and with the fp64 oracle, within the parity tolerances; and record
it into a CUDA graph (where an allocation would fail the capture) and replay
the graph on new inputs copied into the captured tensors.  The file
is named so that pytest collects it last; it also passes alone in a fresh
process.  The refusal of sizes beyond the built-in buffer needs no GPU and is
checked in the CPU tier (tests/test_abi.py).
"""
import ctypes

import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


def _noalloc(dev, wl):
    lib = ssd.lib()
    dims = ssd.make_dims(dev["x"], dev["B"], wl.chunk)
    y = torch.empty_like(dev["x"])
    fin = torch.empty_like(dev["init"])
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    s = lib.ssd_scan_fwd_noalloc(ctypes.byref(dims), p(dev["x"]), p(dev["dt"]), p(dev["A"]), p(dev["B"]),
                                 p(dev["C"]), p(dev["D"]), p(dev["init"]), p(y), p(fin),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return s, y, fin


@pytest.mark.parametrize("name,over", [
    ("tiny_f32", dict(batch=2, seqlen=300, nheads=4, ngroups=2, init_var=0.3)),
    ("mamba2_130m_layer", dict(batch=2, seqlen=1000, nheads=4, ngroups=2, init_var=0.1)),
])
def test_noalloc_matches_unfused_twice(name, over):
    assert torch.cuda.is_available()
    wl = inputs.custom(name, **over)
    for seed in (0, 1):  # two calls in a row; the second must not see the first's scratch
        host = inputs.generate(wl, seed=seed)
        dev = device_inputs(host)
        s, y, fin = _noalloc(dev, wl)
        assert s == 0, ssd.status_string(s)
        y_ref, f_ref = ssd.ssd_scan_fwd_unfused(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                                                dev["init"], chunk=wl.chunk)
        torch.cuda.synchronize()
        assert rel_err(to_np64(y), to_np64(y_ref)) <= TOL[wl.io]
        assert rel_err(to_np64(fin), to_np64(f_ref)) <= TOL[wl.io]
        y64, f64 = oracle.scan_recurrence(*oracle_args(host))
        assert rel_err(to_np64(y), y64) <= TOL[wl.io]
        assert rel_err(to_np64(fin), f64) <= TOL[wl.io]


def test_noalloc_recorded_in_cuda_graph():
    """The call the entry point exists for: inside an open stream capture.  One
    eager call first (the one-time set-up: kernel attributes, the scratch
    address), then the call is captured and the graph replayed on two further
    input sets copied into the same tensors."""
    assert torch.cuda.is_available()
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=1000, nheads=4, ngroups=2, init_var=0.1)
    dev = device_inputs(inputs.generate(wl, seed=0))
    s, _, _ = _noalloc(dev, wl)
    torch.cuda.synchronize()
    assert s == 0, ssd.status_string(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        s, y, fin = _noalloc(dev, wl)
    assert s == 0, ssd.status_string(s)
    for seed in (1, 2):
        host = inputs.generate(wl, seed=seed)
        new = device_inputs(host)
        for k in dev:
            dev[k].copy_(new[k])
        g.replay()
        y_ref, f_ref = ssd.ssd_scan_fwd_unfused(new["x"], new["dt"], new["A"], new["B"], new["C"], new["D"],
                                                new["init"], chunk=wl.chunk)
        torch.cuda.synchronize()
        assert rel_err(to_np64(y), to_np64(y_ref)) <= TOL[wl.io]
        assert rel_err(to_np64(fin), to_np64(f_ref)) <= TOL[wl.io]
        y64, f64 = oracle.scan_recurrence(*oracle_args(host))
        assert rel_err(to_np64(y), y64) <= TOL[wl.io]
        assert rel_err(to_np64(fin), f64) <= TOL[wl.io]
    del g
