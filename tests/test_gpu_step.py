"""Decode step (ssd_step) against the oracle's token recurrence and against
the chunked scan over the same tokens."""
import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [
    ("tiny_f32", dict(batch=2, seqlen=40, nheads=4, ngroups=2, init_var=0.3)),
    ("tiny_f32", dict(batch=1, seqlen=20, nheads=3, ngroups=1, headdim=5, dstate=7, init_var=0.3)),
    ("mamba2_130m_layer", dict(batch=2, seqlen=24, nheads=4, ngroups=2, init_var=0.1)),
    ("mamba2_2p7b_layer", dict(seqlen=6)),
    # staged kernel with 3 column groups (256 threads do not split evenly) and with 1
    ("tiny_f32", dict(batch=2, seqlen=12, nheads=2, ngroups=1, headdim=12, dstate=100, init_var=0.3)),
    ("mamba2_130m_layer", dict(batch=1, seqlen=10, nheads=2, ngroups=1, headdim=4, dstate=128, init_var=0.1)),
])
def test_decode_steps_match_oracle(name, over):
    wl = inputs.custom(name, **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    state = dev["init"].clone()
    ys = []
    for t in range(wl.seqlen):
        ys.append(ssd.ssd_step(dev["x"][:, t].contiguous(), dev["dt"][:, t].contiguous(), dev["A"],
                               dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(), state, D=dev["D"]))
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=1)
    assert rel_err(to_np64(y), y_ref) <= TOL[wl.io]
    assert rel_err(to_np64(state), f_ref) <= TOL[wl.io]


def test_decode_continues_a_prefill():
    """Prefill with the chunked scan, then decode: equals one scan over all tokens."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=520, nheads=4, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    L0 = 512
    pre = lambda t: t[:, :L0].contiguous()
    y0, st = ssd.ssd_scan_fwd(pre(dev["x"]), pre(dev["dt"]), dev["A"], pre(dev["B"]), pre(dev["C"]), dev["D"],
                              dev["init"], chunk=wl.chunk)
    ys = [y0]
    for t in range(L0, wl.seqlen):
        ys.append(ssd.ssd_step(dev["x"][:, t].contiguous(), dev["dt"][:, t].contiguous(), dev["A"],
                               dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(), st,
                               D=dev["D"]).unsqueeze(1))
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1)
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(st), f_ref) <= TOL["bf16"]


def test_decode_state_view_not_16_byte_aligned():
    """A state that is only 4-byte aligned (a view one float into a buffer) takes
    the scalar kernel and gives the same results as the staged kernel."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=8, nheads=4, ngroups=2, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    n = dev["init"].numel()
    buf = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    st_u = buf[1:].view(dev["init"].shape)
    st_u.copy_(dev["init"])
    st_a = dev["init"].clone()
    for t in range(wl.seqlen):
        args = (dev["x"][:, t].contiguous(), dev["dt"][:, t].contiguous(), dev["A"], dev["B"][:, t].contiguous(),
                dev["C"][:, t].contiguous())
        ya = ssd.ssd_step(*args, st_a, D=dev["D"])
        yu = ssd.ssd_step(*args, st_u, D=dev["D"])
        torch.cuda.synchronize()
        assert rel_err(to_np64(yu), to_np64(ya)) <= 1e-6
    assert rel_err(to_np64(st_u), to_np64(st_a)) <= 1e-6
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(st_u), f_ref) <= TOL["bf16"]
