"""Seeded synthetic inputs for the chunked SSD scan.

This module draws inputs only; it contains none of the scan's arithmetic.
The fp64 oracle (through the tests) and the CUDA path both consume the arrays
it returns.  The generator itself is C (``ssdgen.c``): a counter-based
splitmix64 stream per tensor, so any slice is reproducible on its own and
the values do not depend on the thread count.

Workloads (distributions per tensor; "N(0, v)" means variance v):

=====================  ==================================================
tiny_f32               B1 L256 H2 P16 N16 G1 Q64, fp32 io
mamba2_130m_layer      B2 L4096 H24 P64 N128 G1 Q256, bf16 io
mamba2_2p7b_layer      B8 L16384 H80 P64 N128 G1 Q256, bf16 io, h0 ~ N(0, 0.1)
long_context_layer     B1 L131072 H80 P64 N128 G8 Q256, bf16 io, slow decay
stack24_vertical       B2 L65536 H24 P64 N128 G1 Q256 V2048, 24 layers
=====================  ==================================================

x ~ N(0, 1); dt = softplus(N(0, 1) + shift) with shift -2 (-4 for the long
context layer); A_h = -exp(U[0, ln 16]); B, C ~ N(0, 1/N) shared by the heads
of a group; D = 0 for the tiny case, D_h ~ N(0, 1) otherwise; initial state
zero except the 2.7B-shaped layer (N(0, 0.1)).  Every tensor has its own
stream keyed by (seed, workload id, layer, tensor id).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, replace, asdict
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssdgen.c")
_LIB_PATH = os.path.join(_HERE, "libssdgen.so")

# tensor ids used in the stream keys
TENSOR_IDS = {"x": 0, "dt": 1, "A": 2, "B": 3, "C": 4, "D": 5, "init": 6, "Av": 7}

NORMAL, UNIFORM, SOFTPLUS_NORMAL, NEG_EXP_UNIFORM, CONSTANT = 0, 1, 2, 3, 4


def build_lib(force: bool = False) -> str:
    """Compile ssdgen.c into libssdgen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        build_lib()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.ssdgen_key.restype = ctypes.c_uint64
        lib.ssdgen_key.argtypes = [ctypes.c_uint64] * 4
        lib.ssdgen_fill.restype = None
        lib.ssdgen_fill.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        lib.ssdgen_fill_indexed.restype = None
        lib.ssdgen_fill_indexed.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_int64, ctypes.c_uint64, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_double]
        lib.ssdgen_raw_u64.restype = None
        lib.ssdgen_raw_u64.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int            # workload id, part of every stream key
    batch: int
    seqlen: int
    nheads: int
    headdim: int        # P
    dstate: int         # N
    ngroups: int        # G
    chunk: int          # Q
    io: str             # "f32" or "bf16": dtype of x, B, C, y
    dt_shift: float = -2.0
    d_normal: bool = True      # D_h ~ N(0,1) if True else D = 0
    init_var: float = 0.0      # variance of the initial state (0 => zeros)
    n_layers: int = 1
    vblock: Optional[int] = None

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def dims(self) -> dict:
        return asdict(self)


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", 0, 1, 256, 2, 16, 16, 1, 64, "f32", d_normal=False),
    "mamba2_130m_layer": Workload("mamba2_130m_layer", 1, 2, 4096, 24, 64, 128, 1, 256, "bf16"),
    "mamba2_2p7b_layer": Workload("mamba2_2p7b_layer", 2, 8, 16384, 80, 64, 128, 1, 256, "bf16",
                                  init_var=0.1),
    "long_context_layer": Workload("long_context_layer", 3, 1, 131072, 80, 64, 128, 8, 256, "bf16",
                                   dt_shift=-4.0),
    "stack24_vertical": Workload("stack24_vertical", 4, 2, 65536, 24, 64, 128, 1, 256, "bf16",
                                 n_layers=24, vblock=2048),
}


def custom(base: str = "tiny_f32", **overrides) -> Workload:
    """A workload with the distributions of `base` and changed sizes."""
    return replace(WORKLOADS[base], **overrides)


def stream_key(seed: int, wid: int, layer: int, tensor: str) -> int:
    return int(_load().ssdgen_key(seed, wid, layer, TENSOR_IDS[tensor]))


def fill(shape, io: str, key: int, dist: int, p0: float, p1: float, first: int = 0) -> np.ndarray:
    """Draw a contiguous array of `shape`; io 'f32' -> float32, 'bf16' -> uint16 bit patterns."""
    n = int(np.prod(shape)) if len(shape) else 1
    if io == "f32":
        out = np.empty(shape, dtype=np.float32)
        code = 0
    elif io == "bf16":
        out = np.empty(shape, dtype=np.uint16)
        code = 1
    else:
        raise ValueError(io)
    if n:
        _load().ssdgen_fill(out.ctypes.data, code, first, n, key, dist, p0, p1)
    return out


def tensor_spec(wl: Workload, name: str):
    """(shape, io, dist, p0, p1) for one input tensor of a workload."""
    Bz, L, H, P, N, G = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    bc_std = 1.0 / math.sqrt(N)
    if name == "x":
        return (Bz, L, H, P), wl.io, NORMAL, 0.0, 1.0
    if name == "dt":
        return (Bz, L, H), "f32", SOFTPLUS_NORMAL, wl.dt_shift, 1.0
    if name == "A":
        return (H,), "f32", NEG_EXP_UNIFORM, 0.0, math.log(16.0)
    if name == "Av":  # the vector-valued decay's rates: one per (head, state channel), as A per head
        return (H, N), "f32", NEG_EXP_UNIFORM, 0.0, math.log(16.0)
    if name in ("B", "C"):
        return (Bz, L, G, N), wl.io, NORMAL, 0.0, bc_std
    if name == "D":
        return ((H,), "f32", NORMAL, 0.0, 1.0) if wl.d_normal else ((H,), "f32", CONSTANT, 0.0, 0.0)
    if name == "init":
        if wl.init_var > 0:
            return (Bz, H, N, P), "f32", NORMAL, 0.0, math.sqrt(wl.init_var)
        return (Bz, H, N, P), "f32", CONSTANT, 0.0, 0.0
    raise KeyError(name)


def generate(wl: Workload, seed: int = 0, layer: int = 0,
             names=("x", "dt", "A", "B", "C", "D", "init")) -> Dict[str, np.ndarray]:
    """Draw the named input tensors of `wl` (layer `layer` for stacks).

    x, B, C come back as float32 (io f32) or uint16 bf16 bit patterns (io bf16);
    dt, A, D, init are float32.
    """
    out = {}
    for name in names:
        shape, io, dist, p0, p1 = tensor_spec(wl, name)
        out[name] = fill(shape, io, stream_key(seed, wl.wid, layer, name), dist, p0, p1)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact fp64 copy of a stored fp32 array or bf16 bit-pattern array."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def raw_u64(key: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().ssdgen_raw_u64(out.ctypes.data, key, first, n)
    return out
