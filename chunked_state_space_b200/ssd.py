"""Python binding of libssd.so: the C-ABI entry points of include/ssd.h under
the same names, taking torch tensors.

This layer only marshals arguments (shapes, dtypes, pointers, the current
CUDA stream) and allocates outputs and workspace with torch; every step of
the scan runs in libssd's CUDA kernels.  If libssd.so is missing or cannot
be loaded, importing a function raises -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
STATUS_NAMES = ["SSD_OK", "SSD_ERR_INVALID_ARG", "SSD_ERR_SHAPE", "SSD_ERR_DTYPE", "SSD_ERR_ALIGN",
                "SSD_ERR_UNSUPPORTED", "SSD_ERR_WORKSPACE", "SSD_ERR_CUDA", "SSD_ERR_TIMEOUT"]

# every symbol include/ssd.h declares
EXPORTED = ["ssd_status_string", "ssd_version", "ssd_scan_workspace_size", "ssd_scan_fwd",
            "ssd_scan_fwd_unfused", "ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing",
            "ssd_chunk_scan", "ssd_rmsnorm", "ssd_vertical_workspace_size", "ssd_vertical_fwd",
            "ssd_read_device_status", "ssd_selftest_umma", "ssd_scan_path", "ssd_step",
            "ssd_selftest_fused_trace", "ssd_scan_fwd_noalloc",
            "ssd_selftest_timeout", "ssd_scan_fwd_host", "ssd_scan_fwd_host_workspace_size",
            "ssd_scan_fwd_strided", "ssd_selftest_carry_timeout", "ssd_scan_fwd_vdecay",
            "ssd_selftest_set_segments", "ssd_selftest_set_split", "ssd_selftest_set_step_chunks",
            "ssd_scan_fwd_normed"]


class SSDError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("chunk", ctypes.c_int64), ("io_dtype", ctypes.c_int32), ("flags", ctypes.c_int32)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_lib = None


def lib() -> ctypes.CDLL:
    """Load libssd.so (raises if it is missing: build it with
    ``python -m chunked_state_space_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libssd.so not found at {LIB_PATH}; run `python -m chunked_state_space_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    D = ctypes.POINTER(Dims)
    sig = {
        "ssd_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "ssd_version": (ctypes.c_int, []),
        "ssd_scan_workspace_size": (ctypes.c_int, [D, ctypes.POINTER(ctypes.c_size_t)]),
        "ssd_scan_fwd": (ctypes.c_int, [D] + [_P] * 10 + [ctypes.c_size_t, _P]),
        "ssd_scan_fwd_unfused": (ctypes.c_int, [D] + [_P] * 10 + [ctypes.c_size_t, _P]),
        "ssd_scan_fwd_host": (ctypes.c_int, [D] + [_P] * 10 + [ctypes.c_size_t, _P]),
        "ssd_scan_fwd_host_workspace_size": (ctypes.c_int, [D, _P]),
        "ssd_scan_fwd_strided": (ctypes.c_int, [D, _P, _I64, _I64, _P, _I64, _I64, _P, _P, _P, _I64, _I64, _P, _P,
                                                _P, _I64, _I64, _P, _P]),
        "ssd_chunk_cumsum": (ctypes.c_int, [D, _P, _P, _P, _P]),
        "ssd_chunk_state": (ctypes.c_int, [D, _P, _P, _P, _P, _P]),
        "ssd_state_passing": (ctypes.c_int, [D, _P, _P, _P, _P, _P, _P]),
        "ssd_chunk_scan": (ctypes.c_int, [D, _P, _P, _P, _P, _P, _P, _P, _P]),
        "ssd_rmsnorm": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _P, ctypes.c_float, _P,
                                       _P]),
        "ssd_vertical_workspace_size": (ctypes.c_int, [D, ctypes.c_int32, ctypes.c_int64,
                                                       ctypes.POINTER(ctypes.c_size_t)]),
        "ssd_vertical_fwd": (ctypes.c_int, [D, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, _P,
                                            _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
        "ssd_read_device_status": (ctypes.c_int, [_P]),
        "ssd_selftest_umma": (ctypes.c_int, [ctypes.c_int32, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P]),
        "ssd_scan_path": (ctypes.c_int, [D, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
        "ssd_step": (ctypes.c_int, [D] + [_P] * 9),
        "ssd_scan_fwd_noalloc": (ctypes.c_int, [D] + [_P] * 10),
        "ssd_selftest_fused_trace": (ctypes.c_int, [D] + [_P] * 10 + [ctypes.c_int64, _P]),
        "ssd_selftest_timeout": (ctypes.c_int, [D] + [_P] * 10),
        "ssd_selftest_carry_timeout": (ctypes.c_int, [D] + [_P] * 10 + [ctypes.c_size_t, _P]),
        "ssd_selftest_set_segments": (ctypes.c_int, [ctypes.c_int]),
        "ssd_selftest_set_split": (ctypes.c_int, [ctypes.c_int, ctypes.c_int64]),
        "ssd_selftest_set_step_chunks": (ctypes.c_int, [ctypes.c_int]),
        "ssd_scan_fwd_normed": (ctypes.c_int, [D, _P, _P, ctypes.c_float] + [_P] * 10),
        "ssd_scan_fwd_vdecay": (ctypes.c_int, [D] + [_P] * 10),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(s: int) -> str:
    return lib().ssd_status_string(s).decode()


def _check(s: int, what: str):
    if s != 0:
        raise SSDError(s, f"{what}: {status_string(s)}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _io_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise SSDError(3, f"unsupported io dtype {t.dtype}")


FLAG_INPUT_DT = 1        # SSD_FLAG_INPUT_DT: the input term is dt_t B_t x_t^T
FLAG_TWO_HEADS_PER_CTA = 2  # SSD_FLAG_TWO_HEADS_PER_CTA: the two-head kernel where it applies


def make_dims(x: torch.Tensor, Bm: torch.Tensor, chunk: int, input_dt: bool = False,
              two_heads: bool = False) -> Dims:
    if x.dim() != 4 or Bm.dim() != 4:
        raise SSDError(2, "x must be [B,L,H,P] and B/C [B,L,G,N]")
    Bz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    flags = (FLAG_INPUT_DT if input_dt else 0) | (FLAG_TWO_HEADS_PER_CTA if two_heads else 0)
    return Dims(Bz, L, H, P, N, G, int(chunk), _io_code(x), flags)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise SSDError(1, "tensors must be contiguous")


PATH_NAMES = {0: "cuda_cores", 1: "tensor_steps", 2: "fused", 3: "fused_pair"}
FUSED_PATHS = ("fused", "fused_pair")


def ssd_scan_path(dims: Dims):
    """(path name, kernel launches per call) that ssd_scan_fwd uses for `dims`."""
    p, k = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().ssd_scan_path(ctypes.byref(dims), ctypes.byref(p), ctypes.byref(k)), "ssd_scan_path")
    return PATH_NAMES[p.value], int(k.value)


def ssd_scan_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ssd_scan_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "ssd_scan_workspace_size")
    return int(n.value)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if workspace is not None:
        return workspace
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def ssd_scan_fwd(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, y=None, final_state=None,
                 workspace=None, stream=None, want_final: bool = True, unfused: bool = False, input_dt: bool = False,
                 two_heads: bool = False):
    """y, final_state = scan(x, dt, A, B, C, D, init_state) with chunk size `chunk`.
    input_dt: the input term is dt_t B_t x_t^T (tensor-core path).
    two_heads: the fused kernel with two heads of a group per CTA where it applies."""
    _contig(x, dt, A, Bm, Cm, D, init_state, y, final_state)
    dims = make_dims(x, Bm, chunk, input_dt, two_heads)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  device=x.device)
    nbytes = ssd_scan_workspace_size(dims)
    ws = _workspace(nbytes, x.device, workspace)
    fn = lib().ssd_scan_fwd_unfused if unfused else lib().ssd_scan_fwd
    s = fn(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(init_state), _ptr(y),
           _ptr(final_state), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "ssd_scan_fwd_unfused" if unfused else "ssd_scan_fwd")
    return y, final_state


def ssd_scan_fwd_normed(x, ss_in, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, rms_eps: float = 1e-6,
                        y=None, ss_out=None, want_sums: bool = True, final_state=None, want_final: bool = True,
                        stream=None, input_dt: bool = False):
    """One layer of a stack with the RMS norm between layers fused: x is the
    previous layer's stored y and ss_in [B,L,H] f32 its per-(token, head) sums
    of squares (None: x used as is).  Returns (y, ss_out [B,L,H] f32 of this
    layer's stored y or None, final_state)."""
    _contig(x, ss_in, dt, A, Bm, Cm, D, init_state, y, ss_out, final_state)
    dims = make_dims(x, Bm, chunk, input_dt)
    if y is None:
        y = torch.empty_like(x)
    if ss_out is None and want_sums:
        ss_out = torch.empty(x.shape[:3], dtype=torch.float32, device=x.device)
    if final_state is None and want_final:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  device=x.device)
    _check(lib().ssd_scan_fwd_normed(ctypes.byref(dims), _ptr(x), _ptr(ss_in), float(rms_eps), _ptr(dt), _ptr(A),
                                     _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(init_state), _ptr(y), _ptr(ss_out),
                                     _ptr(final_state), _stream(stream)), "ssd_scan_fwd_normed")
    return y, ss_out, final_state


def ssd_scan_fwd_vdecay(x, dt, Av, Bm, Cm, D=None, init_state=None, y=None, final_state=None, stream=None,
                        want_final: bool = True):
    """y, final_state of the scan with a per-channel decay a_t[n] = exp(dt_t Av[h, n]),
    Av [H, N] f32 (token recurrence on CUDA cores; fp32 or bf16 io)."""
    _contig(x, dt, Av, Bm, Cm, D, init_state, y, final_state)
    dims = make_dims(x, Bm, 1)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  device=x.device)
    _check(lib().ssd_scan_fwd_vdecay(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(Av), _ptr(Bm), _ptr(Cm), _ptr(D),
                                     _ptr(init_state), _ptr(y), _ptr(final_state), _stream(stream)),
           "ssd_scan_fwd_vdecay")
    return y, final_state


def ssd_scan_fwd_host_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ssd_scan_fwd_host_workspace_size(ctypes.byref(dims), ctypes.byref(n)),
           "ssd_scan_fwd_host_workspace_size")
    return int(n.value)


def ssd_scan_fwd_host(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, y=None, final_state=None,
                      workspace=None, stream=None, want_final: bool = True, device=None, input_dt: bool = False):
    """ssd_scan_fwd on HOST tensors (pinned for overlapped copies): the batch streams
    through a device workspace one sequence at a time.  Returns host (y, final_state);
    they are complete once `stream` (default: the current stream) has finished."""
    for t in (x, dt, A, Bm, Cm, D, init_state, y, final_state):
        if t is not None and t.is_cuda:
            raise SSDError(1, "ssd_scan_fwd_host takes host tensors")
    _contig(x, dt, A, Bm, Cm, D, init_state, y, final_state)
    dims = make_dims(x, Bm, chunk, input_dt)
    pin = x.is_pinned()
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, pin_memory=pin)
    if final_state is None and want_final:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  pin_memory=pin)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = _workspace(ssd_scan_fwd_host_workspace_size(dims), dev, workspace)
    _check(lib().ssd_scan_fwd_host(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                   _ptr(init_state), _ptr(y), _ptr(final_state), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "ssd_scan_fwd_host")
    return y, final_state


def ssd_scan_fwd_strided(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, y=None, final_state=None,
                         stream=None, want_final: bool = True, input_dt: bool = False, two_heads: bool = False):
    """ssd_scan_fwd on strided views (tensor-core path): x [B,L,H,P], dt [B,L,H],
    B/C [B,L,G,N] and y may have any batch and token strides as long as each
    token's heads (groups) are dense, e.g. slices of one fused projection output.
    Bm and Cm must share their strides."""
    if Bm.stride() != Cm.stride():
        raise SSDError(2, "B and C must have the same strides")
    for t, inner in ((x, (x.shape[3], 1)), (Bm, (Bm.shape[3], 1)), (dt, (1,))):
        if tuple(t.stride()[2:]) != inner:
            raise SSDError(2, "each token's heads/groups must be dense")
    _contig(A, D, init_state, final_state)
    dims = make_dims(x, Bm, chunk, input_dt, two_heads)
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    if final_state is None and want_final:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  device=x.device)
    _check(lib().ssd_scan_fwd_strided(ctypes.byref(dims), _ptr(x), x.stride(0), x.stride(1), _ptr(dt), dt.stride(0),
                                      dt.stride(1), _ptr(A), _ptr(Bm), _ptr(Cm), Bm.stride(0), Bm.stride(1), _ptr(D),
                                      _ptr(init_state), _ptr(y), y.stride(0), y.stride(1), _ptr(final_state),
                                      _stream(stream)), "ssd_scan_fwd_strided")
    return y, final_state


def ssd_scan_fwd_unfused(*args, **kw):
    kw["unfused"] = True
    return ssd_scan_fwd(*args, **kw)


def ssd_chunk_cumsum(dt, A, dims: Dims, lam=None, stream=None):
    nc = -(-dims.seqlen // dims.chunk)
    if lam is None:
        lam = torch.empty((dims.batch, dims.nheads, nc, dims.chunk), dtype=torch.float32, device=dt.device)
    _check(lib().ssd_chunk_cumsum(ctypes.byref(dims), _ptr(dt), _ptr(A), _ptr(lam), _stream(stream)),
           "ssd_chunk_cumsum")
    return lam


def ssd_chunk_state(x, Bm, lam, dims: Dims, states=None, stream=None):
    nc = -(-dims.seqlen // dims.chunk)
    if states is None:
        states = torch.empty((dims.batch, dims.nheads, nc, dims.dstate, dims.headdim), dtype=torch.float32,
                             device=x.device)
    _check(lib().ssd_chunk_state(ctypes.byref(dims), _ptr(x), _ptr(Bm), _ptr(lam), _ptr(states), _stream(stream)),
           "ssd_chunk_state")
    return states


def ssd_state_passing(chunk_states, lam, dims: Dims, init_state=None, prev_states=None, final_state=None,
                      stream=None):
    if prev_states is None:
        prev_states = torch.empty_like(chunk_states)
    if final_state is None:
        final_state = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32,
                                  device=chunk_states.device)
    _check(lib().ssd_state_passing(ctypes.byref(dims), _ptr(chunk_states), _ptr(lam), _ptr(init_state),
                                   _ptr(prev_states), _ptr(final_state), _stream(stream)), "ssd_state_passing")
    return prev_states, final_state


def ssd_chunk_scan(x, Bm, Cm, lam, prev_states, dims: Dims, D=None, y=None, stream=None):
    if y is None:
        y = torch.empty_like(x)
    _check(lib().ssd_chunk_scan(ctypes.byref(dims), _ptr(x), _ptr(Bm), _ptr(Cm), _ptr(lam), _ptr(D),
                                _ptr(prev_states), _ptr(y), _stream(stream)), "ssd_chunk_scan")
    return y


def ssd_rmsnorm(inp: torch.Tensor, eps: float, out=None, stream=None):
    """RMS-normalise each token of a [..., H, P] tensor over its last two axes."""
    _contig(inp)
    if out is None:
        out = torch.empty_like(inp)
    F = inp.shape[-1] * inp.shape[-2]
    rows = inp.numel() // F
    _check(lib().ssd_rmsnorm(rows, F, _io_code(inp), _ptr(inp), float(eps), _ptr(out), _stream(stream)),
           "ssd_rmsnorm")
    return out


def ssd_vertical_workspace_size(dims: Dims, n_layers: int, vblock: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ssd_vertical_workspace_size(ctypes.byref(dims), n_layers, vblock, ctypes.byref(n)),
           "ssd_vertical_workspace_size")
    return int(n.value)


def ssd_vertical_fwd(x0, layers: Sequence[dict], states: Sequence[torch.Tensor], vblock: int, chunk: int = 256,
                     rms_eps: float = 1e-6, y_out=None, workspace=None, stream=None, input_dt: bool = False,
                     two_heads: bool = False):
    """Depth-first multi-layer schedule.  layers[l] has dt, A, B, C and optionally D;
    states[l] ([B,H,N,P] f32) holds layer l's initial state and receives its final state."""
    n = len(layers)
    dims = make_dims(x0, layers[0]["B"], chunk, input_dt, two_heads)
    _contig(x0, *[t for p in layers for t in (p["dt"], p["A"], p["B"], p["C"], p.get("D"))], *states)
    if y_out is None:
        y_out = torch.empty_like(x0)
    arr = lambda key: (ctypes.c_void_p * n)(*[(p[key].data_ptr() if p.get(key) is not None else None)
                                              for p in layers])
    st_arr = (ctypes.c_void_p * n)(*[s.data_ptr() for s in states])
    has_d = any(p.get("D") is not None for p in layers)
    nbytes = ssd_vertical_workspace_size(dims, n, vblock)
    ws = _workspace(nbytes, x0.device, workspace)
    s = lib().ssd_vertical_fwd(ctypes.byref(dims), n, vblock, float(rms_eps), _ptr(x0), arr("dt"), arr("A"),
                               arr("B"), arr("C"), arr("D") if has_d else None, st_arr, _ptr(y_out), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "ssd_vertical_fwd")
    return y_out


def ssd_step(x, dt, A, Bm, Cm, state, D=None, y=None, stream=None, input_dt: bool = False):
    """One decode step: x [B,H,P], dt [B,H], A [H], B/C [B,G,N], state [B,H,N,P] f32
    (updated in place).  Returns y [B,H,P]."""
    _contig(x, dt, A, Bm, Cm, D, state, y)
    Bz, H, P = x.shape
    G, N = Bm.shape[1], Bm.shape[2]
    dims = Dims(Bz, 1, H, P, N, G, 1, _io_code(x), FLAG_INPUT_DT if input_dt else 0)
    if y is None:
        y = torch.empty_like(x)
    _check(lib().ssd_step(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(state),
                          _ptr(y), _stream(stream)), "ssd_step")
    return y


def ssd_read_device_status(stream=None) -> int:
    return int(lib().ssd_read_device_status(_stream(stream)))


def ssd_version() -> int:
    return int(lib().ssd_version())


SELFTEST_VARIANTS = {"A_K_B_K": 0, "A_K_B_MN": 1, "A_MN_B_MN": 2, "A_MN_B_MN_SWAPPED": 3, "TS_A_TMEM_B_MN": 4,
                     "TMA_A_K_B_MN": 5}


def ssd_selftest_umma(variant: str, A: torch.Tensor, B: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    """Diagnostic: D = A_logical[128 x K] @ B_logical[K x N] through tcgen05 with the
    operand layout `variant` (see include/ssd_selftest.h for the storage of A and B)."""
    D = torch.empty((128, N), dtype=torch.float32, device=A.device)
    _check(lib().ssd_selftest_umma(SELFTEST_VARIANTS[variant], _ptr(A), _ptr(B), _ptr(D), N, K, _stream(stream)),
           "ssd_selftest_umma")
    return D


TRACE_EVENTS = ["loads", "S_issued", "c_issued", "mask_start", "mask_done", "lam_ready", "xp_done", "c_seen",
                "state_pub", "epi_done", "c_ready", "c_mid", "S_ready", "mask_ld", "mask_b01", "mask_ld2", "mask_b23",
                "mask_wait_st"]


def ssd_selftest_fused_trace(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, stream=None):
    """Diagnostic: run the fused kernel with CTA 0 tracing its pipeline events.
    Returns (y, final_state, trace [nsub, 24] int64 clocks, ctas [B*H, 3] int64
    (start ns, end ns, SM) of every CTA)."""
    dims = make_dims(x, Bm, chunk)
    nsub = -(-dims.seqlen // 128)
    y = torch.empty_like(x)
    fin = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32, device=x.device)
    ntr = nsub * 24
    trace = torch.zeros(ntr + 3 * dims.batch * dims.nheads, dtype=torch.int64, device=x.device)
    _check(lib().ssd_selftest_fused_trace(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                          _ptr(init_state), _ptr(y), _ptr(fin), _ptr(trace), trace.numel(),
                                          _stream(stream)), "ssd_selftest_fused_trace")
    return y, fin, trace[:ntr].view(nsub, 24), trace[ntr:].view(-1, 3)


def ssd_selftest_timeout(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, stream=None,
                         two_heads: bool = False) -> None:
    """Diagnostic: launch the fused kernel (the two-head one with two_heads, where
    it applies) with its TMA loads withheld, so its bounded waits run out; read
    the outcome with ssd_read_device_status."""
    dims = make_dims(x, Bm, chunk, two_heads=two_heads)
    y = torch.empty_like(x)
    fin = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32, device=x.device)
    _check(lib().ssd_selftest_timeout(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D),
                                      _ptr(init_state), _ptr(y), _ptr(fin), _stream(stream)), "ssd_selftest_timeout")


def ssd_selftest_carry_timeout(x, dt, A, Bm, Cm, D=None, init_state=None, chunk: int = 256, stream=None,
                               two_heads: bool = False) -> None:
    """Diagnostic: launch the fused kernel (the two-head one with two_heads) with
    its split schedule but with no carry ever published, so every wait for one
    runs out; read the outcome with ssd_read_device_status."""
    dims = make_dims(x, Bm, chunk, two_heads=two_heads)
    y = torch.empty_like(x)
    fin = torch.empty((dims.batch, dims.nheads, dims.dstate, dims.headdim), dtype=torch.float32, device=x.device)
    ws = _workspace(ssd_scan_workspace_size(dims), x.device, None)
    _check(lib().ssd_selftest_carry_timeout(ctypes.byref(dims), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm),
                                            _ptr(D), _ptr(init_state), _ptr(y), _ptr(fin), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)),
           "ssd_selftest_carry_timeout")


def ssd_selftest_set_segments(nseg: int) -> None:
    """Segments per sequence of the two-head kernel's schedule for the
    following launches (0 = chosen from the shape)."""
    _check(lib().ssd_selftest_set_segments(int(nseg)), "ssd_selftest_set_segments")


def ssd_selftest_set_split(nseg: int, whole: int) -> None:
    """One-head segmented form for the following launches: the first `whole`
    sequences whole, the rest in about `nseg` segments (nseg 0 = the cost
    model's choice)."""
    _check(lib().ssd_selftest_set_split(int(nseg), int(whole)), "ssd_selftest_set_split")


def ssd_selftest_set_step_chunks(n: int) -> None:
    """Chunks per CTA of the tensor-core step kernels for the following launches
    (0 = chosen from the shape)."""
    _check(lib().ssd_selftest_set_step_chunks(int(n)), "ssd_selftest_set_step_chunks")
