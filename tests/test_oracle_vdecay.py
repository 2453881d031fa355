"""Pins of the oracle's vector-valued-decay variant (scan_recurrence_vdecay,
scan_chunked_vdecay): a_t[n] = exp(dt_t Av[h, n]), one decay rate per state
channel n -- the diagonal state matrix of the selective scan
("告别Transformer的二次方噩梦…" §2.1) and the per-channel decay of the
recurrences "分块推理…" §6 lists (RWKV, xLSTM).

Each pin is independent of the function it checks: a hand-worked example, the
reduction to the (separately pinned) scalar-decay oracle when every channel
has the same rate, prefix sums when nothing decays, an O(L^2) double sum with
explicit per-channel products, and chunked == recurrence for several Q.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = np.array([float(t) for t in v])
    return vals


def problem(Bz=2, L=29, H=4, P=3, N=5, G=2, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bz, L, H, P))
    dt = np.log1p(np.exp(rng.standard_normal((Bz, L, H)) - 1.0))
    Av = -np.exp(rng.uniform(0, math.log(8.0), (H, N)))
    Bm = rng.standard_normal((Bz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bz, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal(H)
    init = 0.3 * rng.standard_normal((Bz, H, N, P))
    return x, dt, Av, Bm, Cm, D, init


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def test_golden_vector_decay():
    g = _read_golden("vector_decay.txt")
    L, N = 3, 2
    x = g["x"].reshape(1, L, 1, 1)
    dt = g["dt"].reshape(1, L, 1)
    Av = g["Av"].reshape(1, N)
    Bm = g["B"].reshape(1, L, 1, N)
    Cm = g["C"].reshape(1, L, 1, N)
    init = g["h0"].reshape(1, 1, N, 1)
    y, fin = oracle.scan_recurrence_vdecay(x, dt, Av, Bm, Cm, g["D"], init)
    assert np.allclose(y.ravel(), g["y"], rtol=0, atol=1e-12)
    assert np.allclose(fin.ravel(), g["final"], rtol=0, atol=1e-12)
    for Q in (1, 2, 3):
        yc, fc = oracle.scan_chunked_vdecay(x, dt, Av, Bm, Cm, Q, g["D"], init)
        assert np.allclose(yc.ravel(), g["y"], rtol=0, atol=1e-12)
        assert np.allclose(fc.ravel(), g["final"], rtol=0, atol=1e-12)
    # the rates belong to channels: swapping them changes the result
    ys, _ = oracle.scan_recurrence_vdecay(x, dt, Av[:, ::-1].copy(), Bm, Cm, g["D"], init)
    assert np.max(np.abs(ys.ravel() - g["y"])) > 0.5


def test_equal_rates_reduce_to_the_scalar_decay():
    x, dt, Av, Bm, Cm, D, init = problem()
    A = Av[:, 0].copy()
    Av_eq = np.repeat(A[:, None], Av.shape[1], axis=1)
    y, fin = oracle.scan_recurrence_vdecay(x, dt, Av_eq, Bm, Cm, D, init)
    ys, fs = oracle.scan_recurrence(x, dt, A, Bm, Cm, D, init)
    assert rel(y, ys) < 1e-13 and rel(fin, fs) < 1e-13


def test_no_decay_gives_prefix_sums():
    x, dt, Av, Bm, Cm, D, init = problem(seed=1)
    y, fin = oracle.scan_recurrence_vdecay(x, dt, np.zeros_like(Av), Bm, Cm, D, init)
    Bz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    g = np.arange(H) // (H // G)
    outer = np.einsum("blhn,blhp->blhnp", Bm[:, :, g], x)         # B_t x_t^T per head
    h = init[:, None] + np.cumsum(outer, axis=1)                   # [B, L, H, N, P]
    y_ref = np.einsum("blhn,blhnp->blhp", Cm[:, :, g], h) + D[None, None, :, None] * x
    assert rel(y, y_ref) < 1e-12 and rel(fin, h[:, -1]) < 1e-12


def test_brute_force_double_sum():
    x, dt, Av, Bm, Cm, D, init = problem(Bz=1, L=17, H=2, P=2, N=3, G=1, seed=2)
    Bz, L, H, P = x.shape
    N = Bm.shape[3]
    y, _ = oracle.scan_recurrence_vdecay(x, dt, Av, Bm, Cm, D, init)
    y_ref = np.zeros_like(y)
    for h in range(H):
        a = np.exp(dt[0, :, h][:, None] * Av[h][None, :])  # [L, N]
        for t in range(L):
            for n in range(N):
                lead = np.prod(a[: t + 1, n])
                acc = lead * init[0, h, n]
                for s in range(t + 1):
                    acc = acc + np.prod(a[s + 1: t + 1, n]) * Bm[0, s, 0, n] * x[0, s, h]
                y_ref[0, t, h] += Cm[0, t, 0, n] * acc
            y_ref[0, t, h] += D[h] * x[0, t, h]
    assert rel(y, y_ref) < 1e-12


@pytest.mark.parametrize("Q", [1, 2, 5, 16, 29, 64])
def test_chunked_equals_recurrence(Q):
    x, dt, Av, Bm, Cm, D, init = problem(seed=3)
    y, fin = oracle.scan_recurrence_vdecay(x, dt, Av, Bm, Cm, D, init)
    yc, fc = oracle.scan_chunked_vdecay(x, dt, Av, Bm, Cm, Q, D, init)
    assert rel(yc, y) < 1e-12 and rel(fc, fin) < 1e-12
