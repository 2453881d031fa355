"""ssd_scan_fwd_host: the scan from and to host memory, copies overlapped with
the scan in slices of one sequence and up to 4096 tokens, the state carried
from slice to slice.  Its results must equal ssd_scan_fwd's on the same
inputs bitwise where a sequence is one slice (the same kernels run every
(batch, head) sequence), and the oracle's within the io dtype's tolerance
(also where sequences are cut into several slices)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


def host_inputs(host: dict, pinned: bool) -> dict:
    out = {}
    for k, v in host.items():
        t = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16 else torch.from_numpy(v)
        out[k] = t.pin_memory() if pinned else t.clone()
    return out


@pytest.mark.parametrize("case", [
    dict(base="mamba2_130m_layer", batch=3, seqlen=1000, nheads=4, ngroups=2, init_var=0.1, pinned=True),
    dict(base="mamba2_130m_layer", batch=2, seqlen=300, nheads=2, pinned=False),
    dict(base="tiny_f32", batch=3, seqlen=300, nheads=4, ngroups=2, init_var=0.5, pinned=True),
])
def test_host_io_matches_device_path(case):
    case = dict(case)
    base, pinned = case.pop("base"), case.pop("pinned")
    wl = inputs.custom(base, **case)
    host = inputs.generate(wl)
    h = host_inputs(host, pinned)
    y_h, f_h = ssd.ssd_scan_fwd_host(h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["init"], chunk=wl.chunk)
    torch.cuda.synchronize()
    dev = device_inputs(host)
    y_d, f_d = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                chunk=wl.chunk)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu())
    assert torch.equal(f_h, f_d.cpu())
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(y_h), y_ref) <= TOL[wl.io]
    assert rel_err(to_np64(f_h), f_ref) <= TOL[wl.io]


def test_host_io_without_optional_tensors():
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=512, nheads=2)
    host = inputs.generate(wl)
    h = host_inputs(host, True)
    y_h, f_h = ssd.ssd_scan_fwd_host(h["x"], h["dt"], h["A"], h["B"], h["C"], None, None, chunk=wl.chunk,
                                     want_final=False)
    torch.cuda.synchronize()
    assert f_h is None
    dev = device_inputs(host)
    y_d, _ = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], None, None, chunk=wl.chunk)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu())


@pytest.mark.parametrize("case", [
    dict(base="mamba2_130m_layer", batch=2, seqlen=10000, nheads=4, ngroups=2, init_var=0.1),  # 3 slices, ragged
    dict(base="tiny_f32", batch=2, seqlen=8200, nheads=2, ngroups=1, init_var=0.5),            # CUDA-core path
])
@pytest.mark.parametrize("want_final", [True, False])
def test_host_io_long_sequences_in_slices(case, want_final):
    """Sequences longer than a slice: several slices per sequence, each scanned
    from the end state of the slice before; y and the final state against the
    oracle and against ssd_scan_fwd (to rounding)."""
    case = dict(case)
    base = case.pop("base")
    wl = inputs.custom(base, **case)
    host = inputs.generate(wl)
    h = host_inputs(host, True)
    y_h, f_h = ssd.ssd_scan_fwd_host(h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["init"], chunk=wl.chunk,
                                     want_final=want_final)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(y_h), y_ref) <= TOL[wl.io]
    if want_final:
        assert rel_err(to_np64(f_h), f_ref) <= TOL[wl.io]
    else:
        assert f_h is None
    dev = device_inputs(host)
    y_d, _ = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk)
    torch.cuda.synchronize()
    assert rel_err(to_np64(y_h), to_np64(y_d.cpu())) <= TOL[wl.io]
