"""The dt-scaled input variant (SSD_FLAG_INPUT_DT): h_t = a_t h_{t-1} +
dt_t B_t x_t^T, y_t = C_t^T h_t + D x_t, on the tensor-core scan, the
vertical schedule and the decode step, against the oracle's recurrence with
the same flag."""
import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_dev, to_np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("over", [
    dict(batch=2, seqlen=1000, nheads=4, ngroups=2, init_var=0.1),
    dict(batch=1, seqlen=300, nheads=2),
    dict(batch=3, seqlen=4096, nheads=8, ngroups=1, init_var=0.1),
])
def test_scan_input_dt_matches_oracle(over):
    wl = inputs.custom("mamba2_130m_layer", **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, input_dt=True)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=True)
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
    # the flag changes the result (the test would not see an ignored flag otherwise)
    y0, _ = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(y0, y_ref) > 1e-2


def test_cuda_core_path_rejects_the_flag():
    wl = inputs.custom("tiny_f32", batch=1, seqlen=64, nheads=2)
    dev = device_inputs(inputs.generate(wl))
    with pytest.raises(ssd.SSDError):
        ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                         chunk=wl.chunk, input_dt=True)


def test_vertical_input_dt_equals_horizontal():
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=1024, nheads=4)
    n_layers, eps, V = 3, 1e-6, 256
    layers = [device_inputs(inputs.generate(wl, layer=l, names=("dt", "A", "B", "C", "D"))) for l in range(n_layers)]
    x0 = to_dev(inputs.generate(wl, names=("x",))["x"])
    zeros = lambda: [torch.zeros((wl.batch, wl.nheads, wl.dstate, wl.headdim), device="cuda") for _ in range(n_layers)]
    st_v = zeros()
    yv = ssd.ssd_vertical_fwd(x0, layers, st_v, vblock=V, chunk=wl.chunk, rms_eps=eps, input_dt=True)
    # horizontal: layer by layer, the norm fused (dt-scaled and normalised input together)
    st_h = zeros()
    x, ss, ys = x0, None, []
    for l, p in enumerate(layers):
        y, ss, _ = ssd.ssd_scan_fwd_normed(x, ss, p["dt"], p["A"], p["B"], p["C"], p["D"], st_h[l], chunk=wl.chunk,
                                           rms_eps=eps, final_state=st_h[l], input_dt=True)
        ys.append(y)
        x = y
    torch.cuda.synchronize()
    assert torch.equal(yv, ys[-1])
    for a, b in zip(st_v, st_h):
        assert torch.equal(a, b)
    # the last layer teacher-forced: the oracle's dt-scaled scan of the previous
    # GPU layer's y, RMS-normalised by the oracle
    host_last = inputs.generate(wl, layer=n_layers - 1, names=("dt", "A", "B", "C", "D"))
    f = inputs.to_f64
    y_ref, _ = oracle.scan_recurrence(oracle.rmsnorm(to_np64(ys[-2]), eps), f(host_last["dt"]), f(host_last["A"]),
                                      f(host_last["B"]), f(host_last["C"]), f(host_last["D"]), None, input_dt=True)
    assert rel_err(to_np64(ys[-1]), y_ref) <= TOL["bf16"]


@pytest.mark.parametrize("name,over", [
    ("tiny_f32", dict(batch=2, seqlen=30, nheads=4, ngroups=2, init_var=0.3)),
    ("mamba2_130m_layer", dict(batch=2, seqlen=20, nheads=4, ngroups=2, init_var=0.1)),
])
def test_decode_input_dt_matches_oracle(name, over):
    wl = inputs.custom(name, **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=True)
    state = dev["init"].clone()
    ys = []
    for t in range(wl.seqlen):
        ys.append(ssd.ssd_step(dev["x"][:, t].contiguous(), dev["dt"][:, t].contiguous(), dev["A"],
                               dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(), state, D=dev["D"],
                               input_dt=True))
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=1)
    assert rel_err(to_np64(y), y_ref) <= TOL[wl.io]
    assert rel_err(to_np64(state), f_ref) <= TOL[wl.io]
