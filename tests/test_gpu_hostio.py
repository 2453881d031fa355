"""ssd_scan_fwd_host: the scan from and to host memory, copies overlapped with
the scan one sequence at a time.  Its results must equal ssd_scan_fwd's on the
same inputs bitwise (the same kernels run every (batch, head) sequence), and
the oracle's within the io dtype's tolerance."""
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
