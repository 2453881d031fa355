"""Sequence sharding across ranks: every rank holds one contiguous token
segment of every sequence (rank r: tokens [r L/N, (r+1) L/N)), the layout of
sequence (context) parallelism.

The chunked scan's inter-chunk recursion ("分块推理…" §2.2: b(c) = b_intra(c) +
(prod a over chunk c) b(c-1)) applies unchanged with a rank's whole segment
as the "chunk":
  1. each rank scans its segment from a zero state (rank 0 from the caller's
     initial state) and keeps the end state F_r and the segment's total
     log-decay lam_r[b, h] = A_h sum_t dt[b, t, h];
  2. the ranks all-gather (F_r, lam_r) -- the one exchange step -- and each
     rank combines them in rank order, S_r = F_r + exp(lam_r) S_{r-1}
     (S_{-1} = 0), which gives its incoming state b_in = S_{r-1};
  3. each rank scans its segment again from b_in: its outputs and (on the
     last rank) the sequence's final state are those of the unsplit scan, up
     to rounding.
Step 3 repeats step 1's work (the scan is run twice); the exchange is one
all-gather of B*H*(N*P + 1) floats per rank.  The scans run in libssd's
kernels; this module only moves the carries between ranks and combines them.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


def segment_log_decay(dt: torch.Tensor, A: torch.Tensor) -> torch.Tensor:
    """lam[b, h] = A_h * sum over the segment's tokens of dt[b, t, h], the log
    of the product of the decays a_t over the segment (in dt's dtype)."""
    return dt.sum(dim=1) * A.to(dt.dtype)[None, :]


def combine_carries(local_final: torch.Tensor, log_decay: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's (end state from its own start state, segment
    log-decay) and return this rank's incoming state S_{r-1}, with
    S_k = F_k + exp(lam_k) S_{k-1} and S_{-1} = 0 (rank 0 gets zeros: its
    start state is the caller's, already inside its F_0).

    local_final [B, H, N, P] f32, log_decay [B, H] f32, on the rank's device
    (CPU tensors for gloo).  Every rank must call it (a collective)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    finals = [torch.empty_like(local_final) for _ in range(world)]
    decays = [torch.empty_like(log_decay) for _ in range(world)]
    dist.all_gather(finals, local_final.contiguous(), group=group)
    dist.all_gather(decays, log_decay.contiguous(), group=group)
    s = torch.zeros_like(local_final)
    for k in range(rank):  # inclusive states of ranks 0 .. rank-1, in order
        s = finals[k] + torch.exp(decays[k])[:, :, None, None] * s
    return s


def ssd_scan_fwd_seqshard(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, group=None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """The scan of this rank's token segment of every sequence, with the state
    handed across the segments of all ranks (see the module docstring).

    x [B, Ls, H, P], dt [B, Ls, H], Bm/Cm [B, Ls, G, N]: this rank's segment;
    A, D [H]; init_state [B, H, N, P] or None: the sequences' initial state
    (read on rank 0 only).  Returns (y [B, Ls, H, P], final [B, H, N, P]): y of
    this segment, and the state after this segment (the sequences' final
    state on the last rank)."""
    from chunked_state_space_b200 import ssd

    rank = dist.get_rank(group)
    start = init_state if rank == 0 else None
    _, local_final = ssd.ssd_scan_fwd(x, dt, A, Bm, Cm, D, start, chunk=chunk, workspace=workspace, stream=stream)
    b_in = combine_carries(local_final, segment_log_decay(dt, A), group)
    if rank == 0:
        b_in = init_state
    return ssd.ssd_scan_fwd(x, dt, A, Bm, Cm, D, b_in, chunk=chunk, workspace=workspace, stream=stream)
