"""fp64 CPU oracle for the chunked SSD scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  It shares no
code with the CUDA path; the two meet only through the seeded arrays of
``chunked_state_space_b200.inputs``.

Functions and the passages they follow (page titles as published):

* ``scan_recurrence``  -- the token recurrence h_t = a_t h_{t-1} + B_t x_t^T,
  y_t = C_t^T h_t + D x_t ("分块推理：解锁循环模型并行计算，实现长序列高效处理" §2;
  per-token dt, B, C: "告别Transformer的二次方噩梦…" §2.1).
* ``scan_chunked``     -- the chunk decomposition with its intermediates
  (by_intra, b_intra, b(c), by_inter; same page §2.1-§2.2).
* ``scan_recurrence_vdecay`` / ``scan_chunked_vdecay`` -- the same with a
  vector-valued decay, one rate per state channel (the diagonal A of the
  selective scan, "告别Transformer的二次方噩梦…" §2.1; per-channel decays as in
  the recurrences of "分块推理…" §6): the token recurrence and its chunk
  decomposition.
* ``round_bf16``, ``rmsnorm``, ``rmsnorm_bf16`` -- storage rounding and the
  layer-to-layer normalisation of the multi-layer stack, unrounded (as a
  fused implementation feeds it) and stored in bf16 (a reading; the page's §3
  only says that layer l's output feeds layer l+1).
* ``stack_horizontal`` / ``stack_vertical`` -- the two multi-layer schedules
  of §3.1 and §3.2 of the same page.

All of them are pinned in tests/test_oracle.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB, defines: Sequence[str] = ()) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=gnu11", "-fno-fast-math",
               "-ffp-contract=off"]
        cmd += [f"-D{d}" for d in defines]
        cmd += ["-o", tmp, src, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, out)
    return out


_P = ctypes.c_void_p
_I = ctypes.c_int64


class _Oracle:
    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_scan_recurrence.restype = None
        lib.oracle_scan_recurrence.argtypes = [_I] * 6 + [_P] * 9 + [ctypes.c_int]
        lib.oracle_scan_chunked.restype = None
        lib.oracle_scan_chunked.argtypes = [_I] * 7 + [_P] * 14 + [ctypes.c_int]
        lib.oracle_scan_recurrence_vdecay.restype = None
        lib.oracle_scan_recurrence_vdecay.argtypes = [_I] * 6 + [_P] * 9
        lib.oracle_scan_chunked_vdecay.restype = None
        lib.oracle_scan_chunked_vdecay.argtypes = [_I] * 7 + [_P] * 9
        lib.oracle_round_bf16.restype = None
        lib.oracle_round_bf16.argtypes = [_I, _P, _P]
        lib.oracle_rmsnorm_bf16.restype = None
        lib.oracle_rmsnorm_bf16.argtypes = [_I, _I, _P, ctypes.c_double, _P]
        lib.oracle_rmsnorm.restype = None
        lib.oracle_rmsnorm.argtypes = [_I, _I, _P, ctypes.c_double, _P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        self.lib = lib


_default: Optional[_Oracle] = None


def load(path: Optional[str] = None) -> _Oracle:
    """Load the default oracle (building it if needed) or one at `path`."""
    global _default
    if path is not None:
        return _Oracle(path)
    if _default is None:
        _default = _Oracle(build())
    return _default


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _dims(x, Bm):
    Bz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert Bm.shape[:2] == (Bz, L) and H % G == 0
    return Bz, L, H, P, N, G


def num_threads(o: Optional[_Oracle] = None) -> int:
    return int((o or load()).lib.oracle_num_threads())


def scan_recurrence(x, dt, A, Bm, Cm, D=None, init=None, want_final=True, o: Optional[_Oracle] = None,
                    input_dt: bool = False):
    """Token-by-token fp64 recurrence.  Returns (y [B,L,H,P], final [B,H,N,P] or None).
    input_dt: the input term is dt_t B_t x_t^T (the skip keeps D x_t)."""
    o = o or load()
    x, dt, A, Bm, Cm, D, init = map(_f64, (x, dt, A, Bm, Cm, D, init))
    Bz, L, H, P, N, G = _dims(x, Bm)
    y = np.empty((Bz, L, H, P))
    fin = np.empty((Bz, H, N, P)) if want_final else None
    o.lib.oracle_scan_recurrence(Bz, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm),
                                 _ptr(D), _ptr(init), _ptr(y), _ptr(fin), int(bool(input_dt)))
    return y, fin


def scan_chunked(x, dt, A, Bm, Cm, Q, D=None, init=None, o: Optional[_Oracle] = None,
                 input_dt: bool = False) -> dict:
    """Chunked fp64 evaluation with every intermediate of the decomposition."""
    o = o or load()
    x, dt, A, Bm, Cm, D, init = map(_f64, (x, dt, A, Bm, Cm, D, init))
    Bz, L, H, P, N, G = _dims(x, Bm)
    nc = (L + Q - 1) // Q
    out = dict(
        lam=np.empty((Bz, H, nc, Q)),
        chunk_states=np.empty((Bz, H, nc, N, P)),
        prev_states=np.empty((Bz, H, nc, N, P)),
        y_intra=np.empty((Bz, L, H, P)),
        y_inter=np.empty((Bz, L, H, P)),
        y=np.empty((Bz, L, H, P)),
        final=np.empty((Bz, H, N, P)),
    )
    o.lib.oracle_scan_chunked(Bz, L, H, P, N, G, Q, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm),
                              _ptr(D), _ptr(init), _ptr(out["lam"]), _ptr(out["chunk_states"]),
                              _ptr(out["prev_states"]), _ptr(out["y_intra"]), _ptr(out["y_inter"]),
                              _ptr(out["y"]), _ptr(out["final"]), int(bool(input_dt)))
    return out


def scan_recurrence_vdecay(x, dt, Av, Bm, Cm, D=None, init=None, o: Optional[_Oracle] = None):
    """Token recurrence with a per-channel decay a_t[n] = exp(dt_t Av[h, n]), Av [H, N].
    Returns (y [B,L,H,P], final [B,H,N,P])."""
    o = o or load()
    x, dt, Av, Bm, Cm, D, init = map(_f64, (x, dt, Av, Bm, Cm, D, init))
    Bz, L, H, P, N, G = _dims(x, Bm)
    assert Av.shape == (H, N)
    y = np.empty((Bz, L, H, P))
    fin = np.empty((Bz, H, N, P))
    o.lib.oracle_scan_recurrence_vdecay(Bz, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(Av), _ptr(Bm), _ptr(Cm),
                                        _ptr(D), _ptr(init), _ptr(y), _ptr(fin))
    return y, fin


def scan_chunked_vdecay(x, dt, Av, Bm, Cm, Q, D=None, init=None, o: Optional[_Oracle] = None):
    """Chunk decomposition of the per-channel-decay scan.  Returns (y, final)."""
    o = o or load()
    x, dt, Av, Bm, Cm, D, init = map(_f64, (x, dt, Av, Bm, Cm, D, init))
    Bz, L, H, P, N, G = _dims(x, Bm)
    assert Av.shape == (H, N)
    y = np.empty((Bz, L, H, P))
    fin = np.empty((Bz, H, N, P))
    o.lib.oracle_scan_chunked_vdecay(Bz, L, H, P, N, G, Q, _ptr(x), _ptr(dt), _ptr(Av), _ptr(Bm), _ptr(Cm),
                                     _ptr(D), _ptr(init), _ptr(y), _ptr(fin))
    return y, fin


def round_bf16(a, o: Optional[_Oracle] = None) -> np.ndarray:
    o = o or load()
    a = _f64(a)
    out = np.empty_like(a)
    o.lib.oracle_round_bf16(a.size, _ptr(a), _ptr(out))
    return out


def rmsnorm(a, eps: float, o: Optional[_Oracle] = None) -> np.ndarray:
    """RMS-normalise each token of a [B, L, H, P] array over its H*P features (fp64, unrounded)."""
    o = o or load()
    a = _f64(a)
    Bz, L, H, P = a.shape
    out = np.empty_like(a)
    o.lib.oracle_rmsnorm(Bz * L, H * P, _ptr(a), eps, _ptr(out))
    return out


def rmsnorm_bf16(a, eps: float, o: Optional[_Oracle] = None) -> np.ndarray:
    """RMS-normalise each token of a [B, L, H, P] array over its H*P features; round to bf16."""
    o = o or load()
    a = _f64(a)
    Bz, L, H, P = a.shape
    out = np.empty_like(a)
    o.lib.oracle_rmsnorm_bf16(Bz * L, H * P, _ptr(a), eps, _ptr(out))
    return out


def stack_horizontal(x0, layers: List[dict], eps: float, o: Optional[_Oracle] = None):
    """Layer-major schedule (page 1 §3.1).

    layers[l] holds dt, A, B, C, D (fp64 arrays) and optionally init.  Layer
    l's y is stored in bf16 (its io dtype), normalised, rounded to bf16 and fed
    to layer l+1.  Returns (y of the last layer before storage rounding,
    list of final states).
    """
    x = _f64(x0)
    finals = []
    y = None
    for li, p in enumerate(layers):
        y, fin = scan_recurrence(x, p["dt"], p["A"], p["B"], p["C"], p.get("D"), p.get("init"), o=o)
        finals.append(fin)
        if li + 1 < len(layers):
            x = rmsnorm_bf16(round_bf16(y, o=o), eps, o=o)
    return y, finals


def stack_vertical(x0, layers: List[dict], eps: float, V: int, o: Optional[_Oracle] = None):
    """Depth-first schedule (page 1 §3.2): each V-token block passes through all
    layers; every layer's state is kept between blocks and used as the next
    block's initial state."""
    x0 = _f64(x0)
    Bz, L, H, P = x0.shape
    N = layers[0]["B"].shape[3]
    states = [None if p.get("init") is None else _f64(p["init"]).copy() for p in layers]
    y_out = np.empty((Bz, L, H, P))
    for k0 in range(0, L, V):
        k1 = min(k0 + V, L)
        x = x0[:, k0:k1]
        for li, p in enumerate(layers):
            y, fin = scan_recurrence(x, p["dt"][:, k0:k1], p["A"], p["B"][:, k0:k1], p["C"][:, k0:k1],
                                     p.get("D"), states[li], o=o)
            states[li] = fin
            if li + 1 < len(layers):
                x = rmsnorm_bf16(round_bf16(y, o=o), eps, o=o)
            else:
                y_out[:, k0:k1] = y
    if any(s is None for s in states):
        raise ValueError("empty sequence")
    return y_out, states
