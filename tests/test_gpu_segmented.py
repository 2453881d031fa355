"""The one-head kernel's segmented form for problems with fewer (batch, head)
sequences than SMs: the segments' end states from a zero start
(k_ssd_segment_states: one accumulated product B^T X'' per segment), their ordered
combine into each segment's start state (the chunk decomposition of
"分块推理…" §2.1-§2.2 with a segment as the chunk), and the full scan of every
segment from its start state.  Compared with the fp64 oracle; the segment
boundaries fall inside the page's Q-token chunks and at ragged ends."""
import contextlib

import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def segments(n):
    ssd.ssd_selftest_set_segments(n)
    try:
        yield
    finally:
        ssd.ssd_selftest_set_segments(0)


def _run(dev, wl, input_dt=False):
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, input_dt=input_dt)
    torch.cuda.synchronize()
    return y, fin


@pytest.mark.parametrize("over,nseg", [
    (dict(batch=2, seqlen=4096, nheads=24, ngroups=1, init_var=0.1), 0),   # the 130M layer: the cost model's choice
    (dict(batch=1, seqlen=1000, nheads=4, ngroups=2, init_var=0.1), 3),    # ragged: 8 sub-chunks in 3 segments
    (dict(batch=2, seqlen=2048, nheads=6, ngroups=3), 16),                 # one sub-chunk per segment
    (dict(batch=1, seqlen=300, nheads=2, ngroups=1, chunk=128, init_var=0.1), 2),  # Q = 128, short last segment
])
@pytest.mark.parametrize("input_dt", [False, True])
def test_segmented_scan_matches_oracle(over, nseg, input_dt):
    wl = inputs.custom("mamba2_130m_layer", **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    with segments(nseg):
        dims = ssd.make_dims(dev["x"], dev["B"], wl.chunk, input_dt)
        path, kernels = ssd.ssd_scan_path(dims)
        assert path == "fused" and kernels == 3  # the segmented form
        y, fin = _run(dev, wl, input_dt)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=input_dt)
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
    assert ssd.ssd_read_device_status() == 0


def test_segmented_and_whole_sequences_agree():
    """The same problem through the segmented form and through one CTA per
    sequence (the strided entry point has no workspace).  Both stay within
    the bf16 bound of the oracle; against each other they differ by bf16
    roundings: a segment's end state takes each input row x_s once rounded
    to bf16 after its decay to the segment's end is folded in, the one-CTA
    scan rounds it after the decay to its 128-token tile's end only, so the
    two sums carry different roundings of the same terms (2^-9 relative
    each)."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=4096, nheads=24, ngroups=1, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y, fin = _run(dev, wl)
    assert ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk))[1] == 3
    ys, fs = ssd.ssd_scan_fwd_strided(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                      chunk=wl.chunk)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    for got_y, got_f in ((y, fin), (ys, fs)):
        assert rel_err(to_np64(got_y), y_ref) <= TOL["bf16"]
        assert rel_err(to_np64(got_f), f_ref) <= TOL["bf16"]
    assert rel_err(to_np64(y), to_np64(ys)) <= 5e-3
    assert rel_err(to_np64(fin), to_np64(fs)) <= 2e-3


@contextlib.contextmanager
def split(nseg, whole):
    ssd.ssd_selftest_set_split(nseg, whole)
    try:
        yield
    finally:
        ssd.ssd_selftest_set_split(0, 0)


@pytest.mark.parametrize("over,nseg,whole", [
    (dict(batch=2, seqlen=1000, nheads=6, ngroups=3, init_var=0.1), 3, 5),   # 7 of 12 sequences segmented, ragged
    (dict(batch=3, seqlen=2048, nheads=4, ngroups=1, init_var=0.1), 16, 11),  # the last one, one sub-chunk per segment
    (dict(batch=1, seqlen=640, nheads=8, ngroups=2, chunk=128), 2, 1),       # all but the first, zero initial state
])
@pytest.mark.parametrize("input_dt", [False, True])
def test_mixed_grid_matches_oracle(over, nseg, whole, input_dt):
    """The mixed layout: the first `whole` sequences scanned whole (from the
    caller's initial state to its final state) and the rest as segments
    (segment end states, combine over the segmented sequences only, segment
    scans), in one grid.  Every sequence of both kinds against the oracle."""
    wl = inputs.custom("mamba2_130m_layer", **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    with split(nseg, whole):
        path, kernels = ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk, input_dt))
        assert path == "fused" and kernels == 3
        y, fin = _run(dev, wl, input_dt)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=input_dt)
    got_y, got_f = to_np64(y), to_np64(fin)
    H = wl.nheads
    for bh in range(wl.batch * H):  # whole and segmented sequences each within the bound
        b, h = divmod(bh, H)
        assert rel_err(got_y[b, :, h], y_ref[b, :, h]) <= TOL["bf16"], (bh, "y")
        assert rel_err(got_f[b, h], f_ref[b, h]) <= TOL["bf16"], (bh, "final state")
    assert ssd.ssd_read_device_status() == 0


def test_partial_round_is_segmented_by_the_cost_model():
    """B*H = one round of CTAs on the SMs plus a few sequences: the cost model
    runs the full round whole and segments the rest (three launches); the
    results equal the oracle and, for the sequences run whole, the
    one-CTA-per-sequence launch bit for bit."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    wl = inputs.custom("mamba2_2p7b_layer", batch=1, seqlen=2048, nheads=sms + 12, ngroups=1, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    assert ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk))[1] == 3
    y, fin = _run(dev, wl)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
    ys, fs = ssd.ssd_scan_fwd_strided(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                      chunk=wl.chunk)
    torch.cuda.synchronize()
    assert torch.equal(y[:, :, :sms], ys[:, :, :sms])
    assert torch.equal(fin[:, :sms], fs[:, :sms])
    assert rel_err(to_np64(y[:, :, sms:]), to_np64(ys[:, :, sms:])) <= 5e-3
    assert ssd.ssd_read_device_status() == 0
