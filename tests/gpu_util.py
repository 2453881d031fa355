"""Helpers shared by the GPU parity tests: seeded inputs on the device, the
oracle on exactly the same stored values, and the parity metric
max|y - y_ref| / max|y_ref|."""
import numpy as np
import torch

import oracle
from chunked_state_space_b200 import inputs

TOL = {"f32": 1e-5, "bf16": 5e-3}


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def device_inputs(host: dict, device="cuda") -> dict:
    return {k: to_dev(v, device) for k, v in host.items()}


def oracle_args(host: dict):
    return [inputs.to_f64(host[k]) for k in ("x", "dt", "A", "B", "C", "D", "init")]


def oracle_sampled(host: dict, wl, pairs):
    """Run the oracle recurrence for a list of (b, h) pairs over the full length.

    The samples are stacked along the head axis of one problem (one head per
    group) so that a single oracle call runs them in parallel.
    Returns y [S, L, P] and final [S, N, P]."""
    hpg = wl.nheads // wl.ngroups
    bs = [b for b, _ in pairs]
    hs = [h for _, h in pairs]
    gs = [h // hpg for h in hs]
    f = inputs.to_f64
    x = np.stack([f(host["x"][b, :, h]) for b, h in pairs], axis=1)[None]        # [1, L, S, P]
    dt = np.stack([f(host["dt"][b, :, h]) for b, h in pairs], axis=1)[None]      # [1, L, S]
    Bm = np.stack([f(host["B"][b, :, g]) for b, g in zip(bs, gs)], axis=1)[None]  # [1, L, S, N]
    Cm = np.stack([f(host["C"][b, :, g]) for b, g in zip(bs, gs)], axis=1)[None]
    A = f(host["A"])[hs]
    D = f(host["D"])[hs]
    init = np.stack([f(host["init"][b, h]) for b, h in pairs])[None]             # [1, S, N, P]
    y, fin = oracle.scan_recurrence(x, dt, A, Bm, Cm, D, init)
    return np.transpose(y[0], (1, 0, 2)), fin[0]
