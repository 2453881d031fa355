"""ssd_scan_fwd_strided: the tensor-core scan on strided views.  x, B and C
are column slices of one fused [B, L, H*P + 2*G*N] projection output, dt a
slice of a wider tensor, y written into a slice of a wider output.  The result
must equal ssd_scan_fwd on contiguous copies bitwise (the same kernel on the
same values), and the output's padding columns must stay untouched."""
import numpy as np
import pytest
import torch

from chunked_state_space_b200 import inputs, ssd
from gpu_util import device_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [
    dict(batch=2, seqlen=1000, nheads=4, ngroups=2, init_var=0.1),
    dict(batch=1, seqlen=513, nheads=8, ngroups=1),
])
def test_strided_views_match_contiguous(case):
    wl = inputs.custom("mamba2_130m_layer", **case)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    Bz, L, H, P, N, G = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    HP, GN = H * P, G * N
    # one fused projection output [x | B | C] per token
    xbc = torch.empty((Bz, L, HP + 2 * GN), dtype=torch.bfloat16, device="cuda")
    xbc[:, :, :HP] = dev["x"].reshape(Bz, L, HP)
    xbc[:, :, HP:HP + GN] = dev["B"].reshape(Bz, L, GN)
    xbc[:, :, HP + GN:] = dev["C"].reshape(Bz, L, GN)
    x = xbc[:, :, :HP].unflatten(2, (H, P))
    Bm = xbc[:, :, HP:HP + GN].unflatten(2, (G, N))
    Cm = xbc[:, :, HP + GN:].unflatten(2, (G, N))
    dtw = torch.zeros((Bz, L, H + 5), dtype=torch.float32, device="cuda")
    dtw[:, :, :H] = dev["dt"]
    dt = dtw[:, :, :H]
    yw = torch.full((Bz, L, HP + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    y = yw[:, :, :HP].unflatten(2, (H, P))
    _, fin = ssd.ssd_scan_fwd_strided(x, dt, dev["A"], Bm, Cm, dev["D"], dev["init"], chunk=wl.chunk, y=y)
    y_ref, f_ref = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                    chunk=wl.chunk)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert torch.equal(fin, f_ref)
    assert torch.all(yw[:, :, HP:] == 7.0)  # the padding columns are untouched
