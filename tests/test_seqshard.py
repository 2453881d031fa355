"""Sequence sharding across ranks (chunked_state_space_b200.seqshard), on CPU
with gloo: world sizes 2 and 3, each rank holding one token segment of every
sequence.  The per-segment scans are the fp64 oracle (test infrastructure);
what is tested is the exchange -- the all-gather of (end state, segment
log-decay) and the in-order combine S_r = F_r + exp(lam_r) S_{r-1} -- against
the unsplit oracle (fp64, so the bound is rounding-level)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _segments(L, world):
    return [(r * L // world, (r + 1) * L // world) for r in range(world)]


def _worker(rank, world, port, L, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from chunked_state_space_b200 import inputs, seqshard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=L, nheads=4, ngroups=2, headdim=8, dstate=16,
                           init_var=0.1)
        host = inputs.generate(wl)
        f = inputs.to_f64
        t0, t1 = _segments(L, world)[rank]
        seg = {k: f(host[k][:, t0:t1]) for k in ("x", "dt", "B", "C")}
        A, D, init = f(host["A"]), f(host["D"]), f(host["init"])
        # 1. local scan of the segment: zero start (rank 0: the sequences' start)
        _, F = oracle.scan_recurrence(seg["x"], seg["dt"], A, seg["B"], seg["C"], D, init if rank == 0 else None)
        # 2. exchange and combine
        lam = seqshard.segment_log_decay(torch.from_numpy(seg["dt"]), torch.from_numpy(A))
        b_in = seqshard.combine_carries(torch.from_numpy(F), lam)
        b_in = init if rank == 0 else b_in.numpy()
        # 3. the segment again from its incoming state
        y, fin = oracle.scan_recurrence(seg["x"], seg["dt"], A, seg["B"], seg["C"], D, b_in)
        q.put((rank, y, fin))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L", [(2, 256), (3, 300), (3, 7)])
def test_sequence_sharded_scan_matches_unsplit_oracle(world, L):
    import oracle
    from chunked_state_space_b200 import inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=L, nheads=4, ngroups=2, headdim=8, dstate=16,
                       init_var=0.1)
    host = inputs.generate(wl)
    f = inputs.to_f64
    y_ref, f_ref = oracle.scan_recurrence(*[f(host[k]) for k in ("x", "dt", "A", "B", "C", "D", "init")])
    y = np.concatenate([r[1] for r in res], axis=1)
    assert np.max(np.abs(y - y_ref)) <= 1e-10 * np.max(np.abs(y_ref))
    assert np.max(np.abs(res[-1][2] - f_ref)) <= 1e-10 * np.max(np.abs(f_ref))
    # the combine is what carries the state: without it (zero start on every
    # rank) the later segments are wrong by O(1)
    t0 = _segments(L, world)[1][0]
    _, F0 = oracle.scan_recurrence(*[f(host[k][:, :t0]) if k in ("x", "dt", "B", "C") else f(host[k])
                                     for k in ("x", "dt", "A", "B", "C", "D", "init")])
    assert np.max(np.abs(F0)) > 1e-3
