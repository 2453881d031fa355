"""The two-heads-per-CTA fused kernel (SSD_FLAG_TWO_HEADS_PER_CTA, path
SSD_PATH_FUSED_PAIR) and its segmented schedule against the fp64 oracle.

Two heads of one group share a CTA, their B/C tiles and S = C B^T.  With the
caller's workspace the kernel can cut every sequence into segments and run the
(segment, sequence) items round-robin on one persistent CTA per SM; a segment
after the first takes its initial state from the CTA that ran the segment
before it (the inter-chunk recursion of "分块推理…" §2.2 handed across CTAs).
The cases cover one pair, ragged and one-token sequences, several pairs per
group, the dt-scaled input, and the segmented schedule with the shape's own
segment count and with forced counts (down to one sub-chunk per segment, and
segments whose predecessor runs in the same round); each is compared with the
oracle at the bf16 tolerance, and the segmented schedule bitwise with whole
sequences (same arithmetic, the carry passes through memory in fp32)."""
import contextlib

import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs, ssd
from gpu_util import TOL, device_inputs, oracle_args, rel_err, to_np64

pytestmark = pytest.mark.gpu


def _scan(dev, wl, **kw):
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, **kw)
    torch.cuda.synchronize()
    return y, fin


@pytest.mark.parametrize("over", [
    dict(batch=1, seqlen=700, nheads=2, ngroups=1, init_var=0.1),     # one pair, ragged tail
    dict(batch=2, seqlen=1, nheads=4, ngroups=2),                      # one token
    dict(batch=2, seqlen=129, nheads=8, ngroups=2, init_var=0.1),      # 4 heads per group, 2 sub-chunks
    dict(batch=1, seqlen=2048, nheads=6, ngroups=3),                   # exact sub-chunks
    dict(batch=1, seqlen=1000, nheads=4, ngroups=1, chunk=128),        # Q = 128
])
@pytest.mark.parametrize("input_dt", [False, True])
def test_pair_kernel_matches_oracle(over, input_dt):
    wl = inputs.custom("mamba2_130m_layer", **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    assert ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk, input_dt, True))[0] == "fused_pair"
    y, fin = _scan(dev, wl, input_dt=input_dt, two_heads=True)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=input_dt)
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
    # the default one-head kernel on the same inputs (both checked against the oracle)
    assert ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk, input_dt))[0] == "fused"
    y1, f1 = _scan(dev, wl, input_dt=input_dt)
    assert rel_err(to_np64(y1), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(f1), f_ref) <= TOL["bf16"]


@contextlib.contextmanager
def segments(n):
    ssd.ssd_selftest_set_segments(n)
    try:
        yield
    finally:
        ssd.ssd_selftest_set_segments(0)


@pytest.mark.parametrize("over,nseg", [
    (dict(batch=2, seqlen=300, nheads=160, ngroups=1, init_var=0.1), 3),   # 160 pairs, one sub-chunk per segment
    (dict(batch=1, seqlen=1000, nheads=300, ngroups=2), 0),                 # 150 pairs, the shape's own choice
    (dict(batch=1, seqlen=1000, nheads=300, ngroups=2), 8),                 # ragged last segment of one sub-chunk
    (dict(batch=3, seqlen=640, nheads=100, ngroups=5, init_var=0.1), 5),    # 150 pairs, 20 heads per group
    (dict(batch=1, seqlen=2048, nheads=8, ngroups=1, init_var=0.1), 16),    # 4 pairs: predecessors in the same round
    (dict(batch=8, seqlen=4096, nheads=80, ngroups=1), 0),                  # 320 pairs of 32 sub-chunks
])
def test_segmented_schedule_matches_oracle_and_whole_sequences(over, nseg):
    wl = inputs.custom("mamba2_130m_layer", **over)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    dims = ssd.make_dims(dev["x"], dev["B"], wl.chunk, two_heads=True)
    assert ssd.ssd_scan_path(dims)[0] == "fused_pair"
    with segments(nseg):
        assert ssd.ssd_scan_workspace_size(dims) > 0  # the schedule is segmented
        y, fin = _scan(dev, wl, two_heads=True)
    if wl.batch * wl.nheads * wl.seqlen <= 2 ** 21:
        y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
        ey, ef = rel_err(to_np64(y), y_ref), rel_err(to_np64(fin), f_ref)
        assert ey <= TOL["bf16"], ey
        assert ef <= TOL["bf16"], ef
    # The carries themselves: the strided entry point has no workspace, so
    # there every CTA runs whole sequences.  The segments must give the same
    # bits (a wrong or late carry changes whole sequences by O(1)).
    ys, fs = ssd.ssd_scan_fwd_strided(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                                      chunk=wl.chunk, two_heads=True)
    torch.cuda.synchronize()
    assert torch.equal(ys, y)
    assert torch.equal(fs, fin)


def test_segmented_schedule_repeatable_and_workspace_reused():
    """Back-to-back calls on one workspace (the carry flags are reset by each
    call) give identical results."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=300, nheads=160, ngroups=1, init_var=0.1)
    dev = device_inputs(inputs.generate(wl))
    dims = ssd.make_dims(dev["x"], dev["B"], wl.chunk, two_heads=True)
    with segments(3):
        ws = torch.empty(ssd.ssd_scan_workspace_size(dims), dtype=torch.uint8, device="cuda")
        ws.fill_(0xFF)  # contents need not be initialised
        outs = [_scan(dev, wl, workspace=ws, two_heads=True) for _ in range(3)]
    for y, f in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(f, outs[0][1])


@pytest.mark.parametrize("two_heads", [False, True])
def test_long_sequences_repeat_bitwise(two_heads):
    """Long runs (512 sub-chunks per sequence) give the same bits every time: a
    race between a kernel's roles (a buffer reused before its last reader
    finished) shows up as run-to-run differences."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=65536, nheads=2, ngroups=1, init_var=0.1)
    dev = device_inputs(inputs.generate(wl))
    outs = [_scan(dev, wl, two_heads=two_heads) for _ in range(4)]
    for y, f in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(f, outs[0][1])
    # and the same bits when the sequence is cut into blocks with the state
    # carried.  With one head per CTA this holds for one CTA per sequence (the
    # strided entry point, no workspace): the segmented form that the
    # workspace entry picks for 4 sequences forms segment end states with
    # their own roundings, so its blocks agree with the whole run to bf16
    # precision (checked below), not bit for bit.
    if two_heads:
        whole = lambda x, dt, B, C, st: ssd.ssd_scan_fwd(x, dt, dev["A"], B, C, dev["D"], st, chunk=wl.chunk,
                                                         final_state=st, two_heads=True)
        ref = outs[0]
    else:
        whole = lambda x, dt, B, C, st: ssd.ssd_scan_fwd_strided(x, dt, dev["A"], B, C, dev["D"], st,
                                                                 chunk=wl.chunk, final_state=st)
        st0 = dev["init"].clone()
        ref = (whole(dev["x"], dev["dt"], dev["B"], dev["C"], st0)[0], st0)
    V = 2048
    y_blk = torch.empty_like(dev["x"])
    st = dev["init"].clone()
    for k0 in range(0, wl.seqlen, V):
        sl = lambda t: t[:, k0:k0 + V].contiguous()
        yk, _ = whole(sl(dev["x"]), sl(dev["dt"]), sl(dev["B"]), sl(dev["C"]), st)
        y_blk[:, k0:k0 + V] = yk
    torch.cuda.synchronize()
    assert torch.equal(y_blk, ref[0])
    assert torch.equal(st, ref[1])
    if not two_heads:  # the segmented whole run against the blocks
        assert rel_err(to_np64(outs[0][0]), to_np64(y_blk)) <= 5e-3
        assert rel_err(to_np64(outs[0][1]), to_np64(st)) <= 2e-3


def test_sequence_shard_single_rank_equals_scan():
    """seqshard on one rank (NCCL, world size 1): the carried state is the
    caller's initial state, so the result is the plain scan's, bitwise."""
    import datetime
    import os
    import torch.distributed as dist
    from chunked_state_space_b200 import seqshard
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=700, nheads=4, ngroups=2, init_var=0.1)
    dev = device_inputs(inputs.generate(wl))
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        y, fin = seqshard.ssd_scan_fwd_seqshard(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                                                dev["init"], chunk=wl.chunk)
        y0, f0 = _scan(dev, wl)
        assert torch.equal(y, y0) and torch.equal(fin, f0)
    finally:
        dist.destroy_process_group()
