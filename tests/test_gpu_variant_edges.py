"""Edge cases of the strided, host-memory and dt-scaled entry points: short
and ragged sequences, one sequence, and the variants combined; each checked
bitwise against the contiguous device scan (same kernel) or against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


def _xbc_views(dev, wl):
    Bz, L, H, P, N, G = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    HP, GN = H * P, G * N
    xbc = torch.empty((Bz, L, HP + 2 * GN), dtype=torch.bfloat16, device="cuda")
    xbc[:, :, :HP] = dev["x"].reshape(Bz, L, HP)
    xbc[:, :, HP:HP + GN] = dev["B"].reshape(Bz, L, GN)
    xbc[:, :, HP + GN:] = dev["C"].reshape(Bz, L, GN)
    return (xbc[:, :, :HP].unflatten(2, (H, P)), xbc[:, :, HP:HP + GN].unflatten(2, (G, N)),
            xbc[:, :, HP + GN:].unflatten(2, (G, N)))


@pytest.mark.parametrize("seqlen", [1, 50, 128, 129, 257])
@pytest.mark.parametrize("input_dt", [False, True])
def test_strided_short_and_ragged(seqlen, input_dt):
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=seqlen, nheads=4, ngroups=2, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    x, Bm, Cm = _xbc_views(dev, wl)
    y, fin = ssd.ssd_scan_fwd_strided(x, dev["dt"], dev["A"], Bm, Cm, dev["D"], dev["init"], chunk=wl.chunk,
                                      input_dt=input_dt)
    y_ref, f_ref = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                    chunk=wl.chunk, input_dt=input_dt)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref) and torch.equal(fin, f_ref)
    yo, fo = oracle.scan_recurrence(*oracle_args(host), input_dt=input_dt)
    assert rel_err(to_np64(y), yo) <= TOL["bf16"] and rel_err(to_np64(fin), fo) <= TOL["bf16"]


@pytest.mark.parametrize("batch,seqlen", [(1, 1), (1, 700), (5, 130)])
@pytest.mark.parametrize("input_dt", [False, True])
def test_host_io_edges(batch, seqlen, input_dt):
    wl = inputs.custom("mamba2_130m_layer", batch=batch, seqlen=seqlen, nheads=4, ngroups=2, init_var=0.1)
    host = inputs.generate(wl)
    h = {}
    for k, v in host.items():
        t = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16 else torch.from_numpy(v)
        h[k] = t.pin_memory()
    y_h, f_h = ssd.ssd_scan_fwd_host(h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["init"], chunk=wl.chunk,
                                     input_dt=input_dt)
    torch.cuda.synchronize()
    dev = device_inputs(host)
    y_d, f_d = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                chunk=wl.chunk, input_dt=input_dt)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu()) and torch.equal(f_h, f_d.cpu())
