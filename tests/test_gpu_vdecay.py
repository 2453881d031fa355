"""The vector-valued-decay scan (ssd_scan_fwd_vdecay: a_t[n] = exp(dt_t Av[h, n]),
one rate per state channel) through the C ABI against the fp64 oracle's
token recurrence: fp32 io at 1e-5, bf16 io at 5e-3, on several shapes
(ragged, one token, groups, init state, P not dividing the thread count) and
with every channel's rate equal, where it must agree with the scalar-decay
scan's oracle too."""
import math

import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


def _av(H, N, seed, equal=False):
    rng = np.random.default_rng(seed)
    if equal:
        return np.repeat((-np.exp(rng.uniform(0, math.log(16.0), H)))[:, None], N, axis=1).astype(np.float32)
    return (-np.exp(rng.uniform(0, math.log(16.0), (H, N)))).astype(np.float32)


@pytest.mark.parametrize("name,over", [
    ("tiny_f32", dict()),
    ("tiny_f32", dict(batch=2, seqlen=300, nheads=4, ngroups=2, init_var=0.3)),
    ("tiny_f32", dict(batch=1, seqlen=1, nheads=2)),
    ("tiny_f32", dict(batch=1, seqlen=45, nheads=3, ngroups=3, headdim=5, dstate=7, init_var=0.3)),
    ("mamba2_130m_layer", dict(batch=2, seqlen=700, nheads=4, ngroups=2, init_var=0.1)),
    ("tiny_f32", dict(batch=1, seqlen=100, nheads=2, headdim=64, dstate=64, init_var=0.3)),  # P 64, fp32 io
    ("mamba2_130m_layer", dict(batch=1, seqlen=37, nheads=3, ngroups=3, dstate=48)),        # P 64, N 48
    ("mamba2_130m_layer", dict(batch=1, seqlen=257, nheads=2, headdim=12, dstate=100, init_var=0.1)),
])
@pytest.mark.parametrize("equal", [False, True])
def test_vdecay_matches_oracle(name, over, equal):
    wl = inputs.custom(name, **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    Av = _av(wl.nheads, wl.dstate, seed=7, equal=equal)
    y, fin = ssd.ssd_scan_fwd_vdecay(dev["x"], dev["dt"], torch.from_numpy(Av).cuda(), dev["B"], dev["C"], dev["D"],
                                     dev["init"])
    torch.cuda.synchronize()
    a = oracle_args(host)
    y_ref, f_ref = oracle.scan_recurrence_vdecay(a[0], a[1], Av.astype(np.float64), a[3], a[4], a[5], a[6])
    assert rel_err(to_np64(y), y_ref) <= TOL[wl.io]
    assert rel_err(to_np64(fin), f_ref) <= TOL[wl.io]
    if equal:  # every channel at the head's rate: the scalar-decay scan's oracle
        ys, fs = oracle.scan_recurrence(a[0], a[1], Av[:, 0].astype(np.float64), a[3], a[4], a[5], a[6])
        assert rel_err(to_np64(y), ys) <= TOL[wl.io]
        assert rel_err(to_np64(fin), fs) <= TOL[wl.io]
