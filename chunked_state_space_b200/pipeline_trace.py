"""Pipeline trace of the fused tensor-core kernel (diagnostics).

    python -m chunked_state_space_b200.pipeline_trace [--workload NAME] [--batch B]

Runs ssd_selftest_fused_trace (the fused kernel with the CTA of batch 0,
head 0 recording the SM clock at each pipeline event of each 128-token
sub-chunk) on a seeded workload and prints the median time between events in
the steady state, which shows the critical path of the per-sub-chunk chain.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from chunked_state_space_b200 import inputs, ssd


def run(workload: str = "mamba2_2p7b_layer", batch: int | None = None, repeats: int = 3) -> np.ndarray:
    wl = inputs.WORKLOADS[workload]
    if batch:
        wl = inputs.custom(wl.name, batch=batch)
    host = inputs.generate(wl)

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    d = {k: dev(v) for k, v in host.items()}
    tr = ctas = None
    for _ in range(repeats):
        _, _, tr, ctas = ssd.ssd_selftest_fused_trace(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init"],
                                                      chunk=wl.chunk)
    torch.cuda.synchronize()
    return tr.cpu().numpy().astype(np.int64), ctas.cpu().numpy().astype(np.int64)


def cta_summary(ctas: np.ndarray) -> dict:
    """Spread of CTA durations and how the launch filled the SMs."""
    t0 = ctas[:, 0].min()
    dur = (ctas[:, 1] - ctas[:, 0]) / 1e3
    return {
        "kernel span us": (ctas[:, 1].max() - t0) / 1e3,
        "CTA duration us (min/median/max)": (dur.min(), float(np.median(dur)), dur.max()),
        "CTAs per SM (max)": int(np.bincount(ctas[:, 2]).max()),
        "SMs used": int(len(np.unique(ctas[:, 2]))),
        "sum of CTA time / (SMs x span)": float(dur.sum() / (len(np.unique(ctas[:, 2])) * (ctas[:, 1].max() - t0) / 1e3)),
    }


def summarize(t: np.ndarray) -> dict:
    n = t.shape[0]
    ss = slice(min(8, n // 4), max(n - 8, n // 4 + 1))
    E = {name: i for i, name in enumerate(ssd.TRACE_EVENTS)}
    med = lambda a: int(np.median(a[ss])) if len(a[ss]) else 0
    out = {
        "period (products issued, j -> j+1)": med(np.diff(t[:, E["c_issued"]])),
        "loads issued -> S ready": med(t[:, E["S_ready"]] - t[:, E["loads"]]),
        "S issued -> mask start": med(t[:, E["mask_start"]] - t[:, E["S_issued"]]),
        "mask start -> mask done": med(t[:, E["mask_done"]] - t[:, E["mask_start"]]),
        "mask done -> products ready": med(t[:, E["c_ready"]] - t[:, E["mask_done"]]),
        "products ready -> issued": med(t[:, E["c_issued"]] - t[:, E["c_ready"]]),
        "products issued -> seen by epilogue": med(t[:, E["c_seen"]] - t[:, E["c_issued"]]),
        "seen -> state published": med(t[:, E["state_pub"]] - t[:, E["c_seen"]]),
        "state published -> epilogue done": med(t[:, E["epi_done"]] - t[:, E["state_pub"]]),
    }
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mamba2_2p7b_layer")
    ap.add_argument("--batch", type=int, default=None)
    args = ap.parse_args()
    t, ctas = run(args.workload, args.batch)
    for k, v in summarize(t).items():
        print(f"{k:40s} {v:8d} clk")
    for k, v in cta_summary(ctas).items():
        print(f"{k:40s} {v}")


if __name__ == "__main__":
    main()
