"""The C-ABI library (CPU only: no kernel is launched here).

Checks that libssd.so loads, exports every function include/ssd.h declares,
and that argument validation rejects bad calls with the documented status
before anything reaches the GPU.  Pointers below are fake addresses: every
call returns from validation before using them.
"""
import ctypes
import os
import re

import pytest

from chunked_state_space_b200 import build as ssd_build
from chunked_state_space_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "ssd_scan_fwd" in names and "ssd_vertical_fwd" in names
    for n in names:
        assert hasattr(lib, n), n
    # the binding knows the same list
    assert set(ssd.EXPORTED) >= set(names)


def test_status_strings_and_version(lib):
    for code, name in enumerate(ssd.STATUS_NAMES):
        assert ssd.status_string(code).startswith(name)
    assert ssd.status_string(99) == "SSD_ERR_UNKNOWN"
    assert ssd.ssd_version() == 100


def dims(**kw):
    d = dict(batch=2, seqlen=1000, nheads=4, headdim=64, dstate=128, ngroups=2, chunk=256, io_dtype=1,
             flags=0)
    d.update(kw)
    return ssd.Dims(**d)


def ws_size(d):
    n = ctypes.c_size_t(0)
    s = ssd.lib().ssd_scan_workspace_size(ctypes.byref(d), ctypes.byref(n))
    return s, n.value


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), 2), (dict(seqlen=0), 2), (dict(nheads=3), 2), (dict(ngroups=0), 2),
    (dict(headdim=65), 5), (dict(dstate=129), 5), (dict(chunk=257), 5), (dict(io_dtype=2), 3),
    (dict(flags=4), 1), (dict(nheads=70000, ngroups=1), 5),
])
def test_workspace_size_rejects(lib, kw, status):
    s, _ = ws_size(dims(**kw))
    assert s == status, ssd.status_string(s)


def test_workspace_size_values(lib):
    s, n = ws_size(dims())
    assert s == 0
    nc = 4
    lam = 2 * 4 * nc * 256 * 4
    states = 2 * 4 * nc * 128 * 64 * 4
    assert n >= lam + states
    assert lib.ssd_scan_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == 1
    assert lib.ssd_scan_workspace_size(ctypes.byref(dims()), None) == 1


# fake, 256-byte aligned device addresses far apart
BASE = 1 << 40
GB = 1 << 30


def call_scan(d, **over):
    ptr = dict(x=BASE, dt=BASE + 2 * GB, A=BASE + 3 * GB, B=BASE + 4 * GB, C=BASE + 5 * GB, D=BASE + 6 * GB,
               init=BASE + 7 * GB, y=BASE + 8 * GB, final=BASE + 9 * GB, ws=BASE + 10 * GB)
    ptr.update(over)
    wsb = over.get("wsbytes", 1 << 40)
    p = lambda k: ctypes.c_void_p(ptr[k]) if ptr[k] is not None else None
    return ssd.lib().ssd_scan_fwd(ctypes.byref(d), p("x"), p("dt"), p("A"), p("B"), p("C"), p("D"), p("init"),
                                  p("y"), p("final"), p("ws"), wsb, None)


@pytest.mark.parametrize("over,status", [
    (dict(x=None), 1), (dict(dt=None), 1), (dict(y=None), 1),
    (dict(x=BASE + 8), 4), (dict(D=BASE + 6 * GB + 4), 4), (dict(final=BASE + 9 * GB + 2), 4),
    (dict(y=BASE + 1024), 1),                     # y overlaps x
    (dict(final=BASE + 7 * GB + 256), 1),         # final partially overlaps init
    (dict(ws=None), 6), (dict(wsbytes=1024), 6), (dict(ws=BASE + 10 * GB + 8), 4),
])
def test_scan_fwd_rejects(lib, over, status):
    s = call_scan(dims(), **over)
    assert s == status, ssd.status_string(s)


def test_scan_fwd_rejects_bad_dims(lib):
    assert call_scan(dims(nheads=5)) == 2
    assert call_scan(dims(io_dtype=7)) == 3
    assert lib.ssd_scan_fwd(None, *([None] * 10), 0, None) == 1


def test_step_entry_points_reject(lib):
    d = dims()
    p = ctypes.c_void_p(BASE)
    assert lib.ssd_chunk_cumsum(ctypes.byref(d), None, p, p, None) == 1
    assert lib.ssd_chunk_cumsum(ctypes.byref(d), ctypes.c_void_p(BASE + 4), p, p, None) == 4
    assert lib.ssd_chunk_state(ctypes.byref(d), p, None, p, p, None) == 1
    assert lib.ssd_state_passing(ctypes.byref(d), p, p, None, None, None, None) == 1
    assert lib.ssd_chunk_scan(ctypes.byref(d), p, p, p, p, None, None, p, None) == 1
    assert lib.ssd_rmsnorm(4, 0, 1, p, 1e-6, p, None) == 2
    assert lib.ssd_rmsnorm(4, 16, 5, p, 1e-6, p, None) == 3
    assert lib.ssd_rmsnorm(4, 16, 1, None, 1e-6, p, None) == 1
    assert lib.ssd_rmsnorm(4, 16, 1, p, -1.0, p, None) == 1


def test_vertical_rejects(lib):
    d = dims()
    n = ctypes.c_size_t(0)
    assert lib.ssd_vertical_workspace_size(ctypes.byref(d), 0, 2048, ctypes.byref(n)) == 2
    assert lib.ssd_vertical_workspace_size(ctypes.byref(d), 3, 0, ctypes.byref(n)) == 2
    assert lib.ssd_vertical_workspace_size(ctypes.byref(d), 3, 512, ctypes.byref(n)) == 0
    one = ctypes.c_size_t(0)
    dv = dims(seqlen=512)
    assert lib.ssd_scan_workspace_size(ctypes.byref(dv), ctypes.byref(one)) == 0
    assert n.value >= one.value + 2 * 2 * 512 * 4 * 64 * 2
    # the wavefront keeps two V-token activation blocks per layer boundary
    act = 2 * 512 * 4 * 64 * 2  # B * V * H * P * bf16 for dims() (batch 2, 4 heads, P 64)
    sizes = {}
    for layers in (1, 2, 3, 24):
        m = ctypes.c_size_t(0)
        assert lib.ssd_vertical_workspace_size(ctypes.byref(d), layers, 512, ctypes.byref(m)) == 0
        sizes[layers] = m.value
    assert sizes[1] == sizes[2] and sizes[2] >= one.value + 2 * act
    sums = 2 * 512 * 4 * 4  # B * V * H f32: the blocks' per-(token, head) sums of squares (fused norm)
    assert sizes[24] - sizes[3] == 2 * (24 - 3) * (act + sums)
    assert lib.ssd_vertical_fwd(ctypes.byref(d), 2, 512, 1e-6, None, *([None] * 6), None, None, 0, None) == 1


def test_normed_entry_rejects(lib):
    """ssd_scan_fwd_normed takes the one-head tensor-core kernel only and checks
    its arguments before anything touches the device (no GPU needed)."""
    f = lib.ssd_scan_fwd_normed
    eps = ctypes.c_float(1e-6)
    d = dims()
    assert f(ctypes.byref(d), *([None] * 2), eps, *([None] * 10)) == 1          # NULL x, dt, ...
    assert f(ctypes.byref(dims(flags=2)), *([None] * 2), eps, *([None] * 10)) == 5  # two heads per CTA
    assert f(ctypes.byref(dims(flags=4)), *([None] * 2), eps, *([None] * 10)) == 1  # unknown flag bit
    assert f(None, *([None] * 2), eps, *([None] * 10)) == 1
    assert f(ctypes.byref(dims(seqlen=0)), *([None] * 2), eps, *([None] * 10)) == 2


def test_host_io_entry_rejects(lib):
    d = dims()
    n = ctypes.c_size_t(0)
    assert lib.ssd_scan_fwd_host_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    one = ctypes.c_size_t(0)
    d1 = dims(batch=1)
    assert lib.ssd_scan_workspace_size(ctypes.byref(d1), ctypes.byref(one)) == 0
    # A, D and two one-sequence buffers (x, y, dt, B, C, init, final) plus scratch
    L, H, P, N, G = 1000, 4, 64, 128, 2
    per_slice = 2 * L * H * P * 2 + L * H * 4 + 2 * L * G * N * 2 + 2 * H * N * P * 4 + one.value
    assert n.value >= 2 * per_slice
    assert lib.ssd_scan_fwd_host_workspace_size(ctypes.byref(d), None) == 1
    assert lib.ssd_scan_fwd_host_workspace_size(ctypes.byref(dims(nheads=5)), ctypes.byref(n)) == 2
    host = ctypes.c_void_p(0x10000)  # never dereferenced: validation returns first
    args = [host] * 5 + [None, None, host, None]
    assert lib.ssd_scan_fwd_host(ctypes.byref(d), None, *args[1:], None, 0, None) == 1       # x NULL
    assert lib.ssd_scan_fwd_host(ctypes.byref(d), *args, None, 0, None) == 6                 # no workspace
    assert lib.ssd_scan_fwd_host(ctypes.byref(d), *args, ctypes.c_void_p(BASE), 1024, None) == 6
    assert lib.ssd_scan_fwd_host(ctypes.byref(d), *args, ctypes.c_void_p(BASE + 8), n.value, None) == 4


def test_strided_entry_rejects(lib):
    d = dims(seqlen=1024, ngroups=1)
    L, H, P, N, G = 1024, 4, 64, 128, 1
    W = H * P + 2 * G * N                      # a fused [x | B | C] row
    f = lambda **kw: lib.ssd_scan_fwd_strided(
        ctypes.byref(kw.get("d", d)), ctypes.c_void_p(kw.get("x", BASE)), kw.get("xb", L * W), kw.get("xt", W),
        ctypes.c_void_p(BASE + 2 * GB), kw.get("dtb", L * H), kw.get("dtt", H), ctypes.c_void_p(BASE + 3 * GB),
        ctypes.c_void_p(BASE + 2 * H * P), ctypes.c_void_p(BASE + 2 * (H * P + G * N)), L * W, W,
        None, None, ctypes.c_void_p(kw.get("y", BASE + 4 * GB)), kw.get("yb", L * H * P), kw.get("yt", H * P),
        None, None)
    assert f(d=dims(headdim=32, seqlen=1024, ngroups=1)) == 5   # tensor-core shapes only
    assert f(xt=H * P - 8) == 2                                  # token stride below a dense row
    assert f(xb=L * W - W) == 2                                  # batch stride below a sequence
    assert f(xt=W + 4, xb=L * (W + 4)) == 4                      # not a multiple of 8 elements
    assert f(x=BASE + 8) == 4                                    # misaligned pointer
    assert f(y=BASE + 2 * H * P) == 1                            # y overlaps the inputs
    assert f(x=0) == 1                                           # NULL x


def test_input_dt_flag_only_on_the_tensor_core_path(lib):
    fl = dict(flags=1)
    # bf16, P 64, N 128, Q 256: the tensor-core path takes it (validation passes; no launch here)
    assert call_scan(dims(**fl), x=None) == 1
    # the CUDA-core path does not take the flag
    assert call_scan(dims(headdim=32, **fl)) == 5
    assert call_scan(dims(io_dtype=0, **fl)) == 5
    d = dims(**fl)
    p = ctypes.c_void_p(BASE)
    assert lib.ssd_chunk_cumsum(ctypes.byref(d), p, p, p, None) == 5
    ptrs = [ctypes.c_void_p(BASE + k * GB) for k in (0, 2, 3, 4, 5, 6, 7, 8, 9, 10)]  # as in call_scan
    assert lib.ssd_scan_fwd_unfused(ctypes.byref(d), *ptrs, 1 << 40, None) == 5


def test_noalloc_rejects_sizes_beyond_its_buffer(lib):
    # The 2.7B-shaped layer needs about 1.4 GB of step-by-step scratch, far beyond
    # the built-in buffer: refused by the size check, before the buffer's device
    # address is looked up and before anything is launched (so no GPU is needed).
    d = dims(batch=8, seqlen=16384, nheads=80, ngroups=1)
    ptrs = [ctypes.c_void_p(BASE + k * (1 << 34)) for k in range(9)]
    assert lib.ssd_scan_fwd_noalloc(ctypes.byref(d), *ptrs, None) == 5
    # a size that fits passes validation; a NULL x is still refused first
    assert lib.ssd_scan_fwd_noalloc(ctypes.byref(dims()), None, *ptrs[1:], None) == 1


def test_vdecay_entry_rejects(lib):
    d = dims(chunk=1)
    ptrs = [ctypes.c_void_p(BASE + k * GB) for k in (0, 2, 3, 4, 5, 6, 7, 8, 9)]  # x dt Av B C D init y final
    assert lib.ssd_scan_fwd_vdecay(ctypes.byref(dims(chunk=1, flags=1)), *ptrs, None) == 5  # no flags
    assert lib.ssd_scan_fwd_vdecay(ctypes.byref(d), ptrs[0], ptrs[1], None, *ptrs[3:], None) == 1  # NULL Av
    assert lib.ssd_scan_fwd_vdecay(ctypes.byref(d), ptrs[0], ptrs[1], ctypes.c_void_p(BASE + 2 * GB + 2),
                                   *ptrs[3:], None) == 4  # Av misaligned
    # y overlapping Av [H, N]
    assert lib.ssd_scan_fwd_vdecay(ctypes.byref(d), *ptrs[:7], ctypes.c_void_p(BASE + 3 * GB + 16), ptrs[8],
                                   None) == 1


def test_selftest_setters_validate_and_reset(lib):
    """The self-test overrides are host state only: negative values are refused,
    zero restores the choice from the shape (no GPU needed)."""
    invalid = ssd.STATUS_NAMES.index("SSD_ERR_INVALID_ARG")
    assert lib.ssd_selftest_set_segments(-1) == invalid
    assert lib.ssd_selftest_set_split(-1, 0) == invalid
    assert lib.ssd_selftest_set_split(0, -1) == invalid
    assert lib.ssd_selftest_set_step_chunks(-1) == invalid
    for n in (3, 0):
        ssd.ssd_selftest_set_segments(n)
        ssd.ssd_selftest_set_split(n, n)
        ssd.ssd_selftest_set_step_chunks(n)
