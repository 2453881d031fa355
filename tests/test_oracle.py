"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself: hand-worked values
(tests/golden), closed forms (a = 1 gives prefix sums, constant a gives
geometric sums), an O(L^2) brute-force unrolling written with numpy, the
invariants the recurrence must satisfy, and the page's claim that the chunked
evaluation loses nothing against the token recurrence ("分块推理：解锁循环模型并行计算，
实现长序列高效处理" §2.3).  tests/test_oracle_mutants.py shows that planted
mistakes in the oracle fail these pins.
"""
import math
import os

import numpy as np
import pytest

import oracle
from chunked_state_space_b200 import inputs

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


def rand_problem(Bz=2, L=37, H=4, P=3, N=5, G=2, seed=0, init=True, D=True, dt_scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bz, L, H, P))
    dt = np.log1p(np.exp(rng.standard_normal((Bz, L, H)) - 1.0)) * dt_scale
    A = -np.exp(rng.uniform(0, math.log(4.0), H))
    Bm = rng.standard_normal((Bz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bz, L, G, N)) / math.sqrt(N)
    Dv = rng.standard_normal(H) if D else None
    h0 = rng.standard_normal((Bz, H, N, P)) if init else None
    return dict(x=x, dt=dt, A=A, Bm=Bm, Cm=Cm, D=Dv, init=h0)


def run_rec(p, o=None):
    return oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], o=o)


def brute_force(p, input_dt=False):
    """y_t = C_t^T[(prod_{r<=t} a_r) h0 + sum_{s<=t}(prod_{r=s+1..t} a_r) u_s B_s x_s^T] + D x_t,
    evaluated as an explicit double sum over (t, s); final state = bracket at t = L-1.
    u_s = dt_s for the dt-scaled input variant, else 1."""
    x, dt, A, Bm, Cm, D, h0 = (p[k] for k in ("x", "dt", "A", "Bm", "Cm", "D", "init"))
    Bz, L, H, P = x.shape
    G, N = Bm.shape[2:]
    y = np.zeros((Bz, L, H, P))
    fin = np.zeros((Bz, H, N, P))
    for b in range(Bz):
        for h in range(H):
            g = h // (H // G)
            a = np.exp(dt[b, :, h] * A[h])
            for t in range(L):
                st = np.zeros((N, P))
                if h0 is not None:
                    st += np.prod(a[: t + 1]) * h0[b, h]
                for s in range(t + 1):
                    u = dt[b, s, h] if input_dt else 1.0
                    st += np.prod(a[s + 1: t + 1]) * u * np.outer(Bm[b, s, g], x[b, s, h])
                y[b, t, h] = Cm[b, t, g] @ st + (D[h] if D is not None else 0.0) * x[b, t, h]
                if t == L - 1:
                    fin[b, h] = st
    return y, fin


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------- hand-worked values

def test_golden_scalar_recurrence():
    g = _read_golden("scalar_recurrence.txt")
    L = len(g["dt"])
    x = g["x"].reshape(1, L, 1, 1)
    dt = g["dt"].reshape(1, L, 1)
    Bm = g["B"].reshape(1, L, 1, 1)
    Cm = g["C"].reshape(1, L, 1, 1)
    y, fin = oracle.scan_recurrence(x, dt, g["A"], Bm, Cm, g["D"], g["h0"].reshape(1, 1, 1, 1))
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fin.ravel(), g["final"], rtol=0, atol=1e-14)
    for Q in (1, 2, 3, 4):
        out = oracle.scan_chunked(x, dt, g["A"], Bm, Cm, Q, g["D"], g["h0"].reshape(1, 1, 1, 1))
        np.testing.assert_allclose(out["y"].ravel(), g["y"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(out["final"].ravel(), g["final"], rtol=0, atol=1e-14)


def test_golden_scalar_recurrence_input_dt():
    g = _read_golden("scalar_recurrence_input_dt.txt")
    L = len(g["dt"])
    x = g["x"].reshape(1, L, 1, 1)
    dt = g["dt"].reshape(1, L, 1)
    Bm = g["B"].reshape(1, L, 1, 1)
    Cm = g["C"].reshape(1, L, 1, 1)
    h0 = g["h0"].reshape(1, 1, 1, 1)
    y, fin = oracle.scan_recurrence(x, dt, g["A"], Bm, Cm, g["D"], h0, input_dt=True)
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fin.ravel(), g["final"], rtol=0, atol=1e-14)
    for Q in (1, 2, 3, 4):
        out = oracle.scan_chunked(x, dt, g["A"], Bm, Cm, Q, g["D"], h0, input_dt=True)
        np.testing.assert_allclose(out["y"].ravel(), g["y"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(out["final"].ravel(), g["final"], rtol=0, atol=1e-14)


def test_golden_outer_product_orientation():
    g = _read_golden("outer_product_orientation.txt")
    N, P = int(g["N"][0]), int(g["P"][0])
    L = 2
    x = g["x"].reshape(1, L, 1, P)
    Bm = g["B"].reshape(1, L, 1, N)
    Cm = g["C"].reshape(1, L, 1, N)
    dt = np.zeros((1, L, 1))
    A = np.array([-1.0])
    y, fin = oracle.scan_recurrence(x, dt, A, Bm, Cm)
    np.testing.assert_array_equal(y.ravel(), g["y"])
    np.testing.assert_array_equal(fin.ravel(), g["final"])
    out = oracle.scan_chunked(x, dt, A, Bm, Cm, 1)
    np.testing.assert_array_equal(out["y"].ravel(), g["y"])
    np.testing.assert_array_equal(out["final"].ravel(), g["final"])


# ---------------------------------------------------------------- closed forms

def test_unit_decay_is_prefix_sum():
    """A = 0 (a = 1): h_t = h0 + sum_{s<=t} B_s x_s^T, an ordinary prefix sum."""
    p = rand_problem(seed=1)
    p["A"] = np.zeros_like(p["A"])
    y, fin = run_rec(p)
    Bz, L, H, P = p["x"].shape
    G = p["Bm"].shape[2]
    grp = np.arange(H) // (H // G)
    outer = np.einsum("blhn,blhp->blhnp", p["Bm"][:, :, grp], p["x"])
    states = p["init"][:, None] + np.cumsum(outer, axis=1)           # [B,L,H,N,P]
    y_ref = np.einsum("blhn,blhnp->blhp", p["Cm"][:, :, grp], states) + p["D"][None, None, :, None] * p["x"]
    assert rel(y, y_ref) < 1e-13
    assert rel(fin, states[:, -1]) < 1e-13


def test_zero_dt_is_prefix_sum():
    p = rand_problem(seed=2, init=False)
    p["dt"] = np.zeros_like(p["dt"])
    y, fin = run_rec(p)
    H = p["x"].shape[2]
    grp = np.arange(H) // (H // p["Bm"].shape[2])
    outer = np.einsum("blhn,blhp->blhnp", p["Bm"][:, :, grp], p["x"])
    assert rel(fin, outer.sum(axis=1)) < 1e-13


def test_constant_decay_geometric_sum():
    """Constant a, B, x: h_t = a^t h0 + (1 - a^t)/(1 - a) B x^T."""
    Bz, L, H, P, N = 1, 50, 3, 4, 6
    rng = np.random.default_rng(3)
    a = np.array([0.9, 0.5, 0.99])
    A = -np.ones(H)
    dt = np.broadcast_to(-np.log(a), (Bz, L, H)).copy()            # dt*A = log a
    bvec = rng.standard_normal(N)
    xvec = rng.standard_normal((H, P))
    Bm = np.broadcast_to(bvec, (Bz, L, 1, N)).copy()
    Cm = rng.standard_normal((Bz, L, 1, N))
    x = np.broadcast_to(xvec, (Bz, L, H, P)).copy()
    h0 = rng.standard_normal((Bz, H, N, P))
    y, fin = oracle.scan_recurrence(x, dt, A, Bm, Cm, None, h0)
    for h in range(H):
        for t in (1, 7, L):
            at = a[h] ** t
            st = at * h0[0, h] + (1 - at) / (1 - a[h]) * np.outer(bvec, xvec[h])
            np.testing.assert_allclose(y[0, t - 1, h], Cm[0, t - 1, 0] @ st, rtol=1e-12, atol=1e-12)
            if t == L:
                np.testing.assert_allclose(fin[0, h], st, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("shape", [
    dict(Bz=1, L=9, H=2, P=3, N=4, G=1),
    dict(Bz=2, L=17, H=4, P=2, N=3, G=2),
    dict(Bz=1, L=23, H=6, P=5, N=2, G=3),
])
def test_brute_force_unrolled(shape):
    p = rand_problem(seed=4, **shape)
    y, fin = run_rec(p)
    yb, fb = brute_force(p)
    assert rel(y, yb) < 1e-12
    assert rel(fin, fb) < 1e-12


# ---------------------------------------------------------------- invariants

def test_linearity_in_x_and_h0():
    p = rand_problem(seed=5)
    q = rand_problem(seed=6)
    q.update(dt=p["dt"], A=p["A"], Bm=p["Bm"], Cm=p["Cm"], D=p["D"])
    r = dict(p)
    r["x"] = 2.0 * p["x"] - 3.0 * q["x"]
    r["init"] = 2.0 * p["init"] - 3.0 * q["init"]
    yp, fp = run_rec(p)
    yq, fq = run_rec(q)
    yr, fr = run_rec(r)
    assert rel(yr, 2 * yp - 3 * yq) < 1e-12
    assert rel(fr, 2 * fp - 3 * fq) < 1e-12


def test_scale_b_and_c_inverse():
    p = rand_problem(seed=7, init=False)
    y, _ = run_rec(p)
    q = dict(p)
    q["Bm"] = p["Bm"] * 4.0
    q["Cm"] = p["Cm"] / 4.0
    y2, _ = run_rec(q)
    assert rel(y2, y) < 1e-13


def test_causality():
    p = rand_problem(seed=8)
    y, _ = run_rec(p)
    t0 = 20
    q = {k: (None if v is None else v.copy()) for k, v in p.items()}
    q["x"][:, t0:] += 5.0
    q["dt"][:, t0:] *= 3.0
    q["Bm"][:, t0:] -= 1.0
    q["Cm"][:, t0:] += 2.0
    y2, _ = run_rec(q)
    np.testing.assert_array_equal(y[:, :t0], y2[:, :t0])
    assert np.max(np.abs(y[:, t0:] - y2[:, t0:])) > 1e-3


def test_split_and_chain():
    p = rand_problem(seed=9, L=41)
    y, fin = run_rec(p)
    for t0 in (1, 13, 40):
        a = {k: v for k, v in p.items()}
        a = dict(p, x=p["x"][:, :t0], dt=p["dt"][:, :t0], Bm=p["Bm"][:, :t0], Cm=p["Cm"][:, :t0])
        ya, fa = run_rec(a)
        b = dict(p, x=p["x"][:, t0:], dt=p["dt"][:, t0:], Bm=p["Bm"][:, t0:], Cm=p["Cm"][:, t0:], init=fa)
        yb, fb = run_rec(b)
        np.testing.assert_array_equal(np.concatenate([ya, yb], axis=1), y)
        np.testing.assert_array_equal(fb, fin)


def test_zero_b_or_c_gives_skip_only():
    p = rand_problem(seed=10, init=False)
    for key in ("Bm", "Cm"):
        q = dict(p)
        q[key] = np.zeros_like(p[key])
        y, _ = run_rec(q)
        np.testing.assert_allclose(y, p["D"][None, None, :, None] * p["x"], rtol=0, atol=0)


# ---------------------------------------------------------------- chunked == recurrence

@pytest.mark.parametrize("L,Q", [(64, 1), (64, 2), (64, 16), (64, 64), (100, 16), (100, 64), (37, 37), (5, 8)])
def test_chunked_matches_recurrence(L, Q):
    p = rand_problem(seed=11, L=L, Bz=2, H=4, P=3, N=5, G=2)
    y, fin = run_rec(p)
    out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], Q, p["D"], p["init"])
    assert rel(out["y"], y) < 1e-12
    assert rel(out["final"], fin) < 1e-12
    # y = by_intra + by_inter + D x
    assert rel(out["y_intra"] + out["y_inter"] + p["D"][None, None, :, None] * p["x"], y) < 1e-12


def test_chunk_intermediates_are_recurrences():
    """by_intra(c) and b_intra(c) are the recurrence on chunk c alone from a zero
    state (page 1 §2.1); prev_states(c) is the recurrence state at the chunk start;
    lam is the cumulative sum of dt*A whose exponential is the running product of a."""
    L, Q = 70, 16
    p = rand_problem(seed=12, L=L, Bz=1, H=2, P=3, N=4, G=1)
    out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], Q, p["D"], p["init"])
    nc = (L + Q - 1) // Q
    for c in range(nc):
        c0, c1 = c * Q, min(c * Q + Q, L)
        sl = slice(c0, c1)
        yc, fc = oracle.scan_recurrence(p["x"][:, sl], p["dt"][:, sl], p["A"], p["Bm"][:, sl], p["Cm"][:, sl])
        assert rel(out["y_intra"][:, sl], yc) < 1e-12
        assert rel(out["chunk_states"][:, :, c], fc) < 1e-12
        if c0 == 0:
            np.testing.assert_array_equal(out["prev_states"][:, :, c], p["init"])
        else:
            _, f0 = oracle.scan_recurrence(p["x"][:, :c0], p["dt"][:, :c0], p["A"], p["Bm"][:, :c0],
                                           p["Cm"][:, :c0], None, p["init"])
            assert rel(out["prev_states"][:, :, c], f0) < 1e-12
        for h in range(2):
            a = np.exp(p["dt"][0, sl, h] * p["A"][h])
            np.testing.assert_allclose(np.exp(out["lam"][0, h, c, : c1 - c0]), np.cumprod(a), rtol=1e-12)
            # padded tail repeats the chunk total
            if c1 - c0 < Q:
                assert np.all(out["lam"][0, h, c, c1 - c0:] == out["lam"][0, h, c, c1 - c0 - 1])


# ---------------------------------------------------------------- bf16 rounding and rmsnorm

def test_round_bf16_matches_torch_on_fp32_values():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(13)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    # exact ties: fp32 values halfway between two bf16 values
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7)], dtype=np.float32)
    v = np.concatenate([v, ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(v.astype(np.float64))
    np.testing.assert_array_equal(got, ref)
    assert got[-3] == 1.0 and got[-2] == 1.0 + 2.0 ** -6 and got[-1] == -2.0


def test_rmsnorm_closed_forms():
    H, P = 3, 4
    F = H * P
    # one-hot row: v / sqrt(v^2/F) = sign(v) sqrt(F) (eps = 0)
    a = np.zeros((1, 2, H, P))
    a[0, 0, 1, 2] = -7.5
    a[0, 1, 0, 0] = 3.0e-3
    out = oracle.rmsnorm_bf16(a, 0.0)
    assert out[0, 0, 1, 2] == oracle.round_bf16(np.array([-math.sqrt(F)]))[0]
    assert out[0, 1, 0, 0] == oracle.round_bf16(np.array([math.sqrt(F)]))[0]
    assert np.count_nonzero(out) == 2
    # scale invariance with eps = 0 and mean square one before rounding
    rng = np.random.default_rng(14)
    b = rng.standard_normal((2, 5, H, P))
    o1 = oracle.rmsnorm_bf16(b, 0.0)
    o2 = oracle.rmsnorm_bf16(b * 1024.0, 0.0)
    np.testing.assert_array_equal(o1, o2)
    ms = np.mean(o1.reshape(10, F) ** 2, axis=1)
    assert np.all(np.abs(ms - 1.0) < 2 * 2.0 ** -8)
    np.testing.assert_array_equal(np.sign(o1), np.sign(b))
    # eps dominates a zero row: stays zero
    assert np.all(oracle.rmsnorm_bf16(np.zeros((1, 1, H, P)), 1e-6) == 0)


def test_rmsnorm_unrounded_closed_forms():
    H, P = 3, 4
    F = H * P
    # one-hot row: v / sqrt(v^2 / F + eps), here with eps = 0.25 worked by hand:
    # v = -7.5 -> v^2 / F = 56.25 / 12 = 4.6875, + 0.25 = 4.9375
    a = np.zeros((1, 1, H, P))
    a[0, 0, 1, 2] = -7.5
    out = oracle.rmsnorm(a, 0.25)
    assert abs(out[0, 0, 1, 2] - (-7.5 / math.sqrt(4.9375))) < 1e-15
    assert np.count_nonzero(out) == 1
    # eps = 0: every row has mean square exactly one, signs kept, scale-free
    rng = np.random.default_rng(15)
    b = rng.standard_normal((2, 5, H, P))
    o1 = oracle.rmsnorm(b, 0.0)
    np.testing.assert_allclose(np.mean(o1.reshape(10, F) ** 2, axis=1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm(b * 1024.0, 0.0), o1, rtol=1e-14, atol=0)
    np.testing.assert_array_equal(np.sign(o1), np.sign(b))
    # one row's features are normalised together, rows independently
    two = np.concatenate([b[:, :1], 3.0 * b[:, :1]], axis=1)
    o2 = oracle.rmsnorm(two, 0.0)
    np.testing.assert_allclose(o2[:, 0], o2[:, 1], rtol=1e-14, atol=0)
    # the stored form is this one rounded to bf16
    np.testing.assert_array_equal(oracle.round_bf16(oracle.rmsnorm(b, 1e-6)), oracle.rmsnorm_bf16(b, 1e-6))


# ---------------------------------------------------------------- multi-layer schedules

def _layers(n_layers, Bz, L, H, P, N, G, seed):
    out = []
    for l in range(n_layers):
        p = rand_problem(Bz=Bz, L=L, H=H, P=P, N=N, G=G, seed=100 + seed + l, init=(l % 2 == 0))
        out.append(dict(dt=p["dt"], A=p["A"], B=p["Bm"], C=p["Cm"], D=p["D"], init=p["init"]))
    return out


@pytest.mark.parametrize("V", [1, 7, 16, 48, 100])
def test_vertical_equals_horizontal(V):
    Bz, L, H, P, N, G = 2, 48, 2, 3, 4, 1
    layers = _layers(3, Bz, L, H, P, N, G, seed=V)
    x0 = oracle.round_bf16(np.random.default_rng(15).standard_normal((Bz, L, H, P)))
    yh, fh = oracle.stack_horizontal(x0, layers, 1e-6)
    yv, fv = oracle.stack_vertical(x0, layers, 1e-6, V)
    np.testing.assert_array_equal(yv, yh)
    for a, b in zip(fv, fh):
        np.testing.assert_array_equal(a, b)


def test_single_layer_stack_is_the_scan():
    Bz, L, H, P, N, G = 1, 30, 2, 3, 4, 2
    layers = _layers(1, Bz, L, H, P, N, G, seed=0)
    x0 = np.random.default_rng(16).standard_normal((Bz, L, H, P))
    y, f = oracle.stack_horizontal(x0, layers, 1e-6)
    l0 = layers[0]
    y2, f2 = oracle.scan_recurrence(x0, l0["dt"], l0["A"], l0["B"], l0["C"], l0["D"], l0["init"])
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(f[0], f2)


def test_two_layer_stack_feeds_normalised_output():
    """Layer 2 of the stack equals a single scan whose input is the stored,
    normalised output of layer 1 (page 1 §3.1: a layer consumes the previous
    layer's output)."""
    Bz, L, H, P, N, G = 1, 25, 2, 3, 4, 1
    layers = _layers(2, Bz, L, H, P, N, G, seed=1)
    x0 = np.random.default_rng(17).standard_normal((Bz, L, H, P))
    y, f = oracle.stack_horizontal(x0, layers, 1e-6)
    l0, l1 = layers
    y1, _ = oracle.scan_recurrence(x0, l0["dt"], l0["A"], l0["B"], l0["C"], l0["D"], l0["init"])
    x1 = oracle.rmsnorm_bf16(oracle.round_bf16(y1), 1e-6)
    assert np.all(oracle.round_bf16(x1) == x1)
    y2, f2 = oracle.scan_recurrence(x1, l1["dt"], l1["A"], l1["B"], l1["C"], l1["D"], l1["init"])
    np.testing.assert_array_equal(y, y2)


# ---------------------------------------------------------------- workload inputs

def test_tiny_workload_chunked_equals_recurrence():
    wl = inputs.WORKLOADS["tiny_f32"]
    t = inputs.generate(wl)
    args = [inputs.to_f64(t[k]) for k in ("x", "dt", "A", "B", "C", "D", "init")]
    y, fin = oracle.scan_recurrence(*args)
    out = oracle.scan_chunked(*args[:5], wl.chunk, args[5], args[6])
    assert rel(out["y"], y) < 1e-12
    assert rel(out["final"], fin) < 1e-12
    assert np.all(np.isfinite(y)) and np.max(np.abs(y)) > 0.1


# ---------------------------------------------------------------- the dt-scaled input variant

def test_input_dt_brute_force():
    """h_t = a_t h_{t-1} + dt_t B_t x_t^T, y_t = C_t^T h_t + D x_t against the explicit double sum."""
    p = rand_problem(seed=11, Bz=2, L=19, H=4, P=3, N=2, G=2)
    y, f = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], input_dt=True)
    yb, fb = brute_force(p, input_dt=True)
    assert rel(y, yb) < 1e-12 and rel(f, fb) < 1e-12
    # the variant differs from the plain scan (the pin would not see a dropped factor otherwise)
    y0, _ = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"])
    assert rel(y, y0) > 1e-3


def test_input_dt_prefix_sum():
    """A = 0 (a = 1): h_t = h0 + sum_{s<=t} dt_s B_s x_s^T, a dt-weighted prefix sum."""
    p = rand_problem(seed=12, Bz=1, L=23, H=2, P=2, N=3, G=1)
    A = np.zeros_like(p["A"])
    y, f = oracle.scan_recurrence(p["x"], p["dt"], A, p["Bm"], p["Cm"], p["D"], p["init"], input_dt=True)
    x, dt, Bm, Cm, D, h0 = p["x"], p["dt"], p["Bm"], p["Cm"], p["D"], p["init"]
    for h in range(2):
        terms = dt[0, :, h, None, None] * Bm[0, :, 0, :, None] * x[0, :, h, None, :]   # [L, N, P]
        st = h0[0, h][None] + np.cumsum(terms, axis=0)
        yy = np.einsum("tn,tnp->tp", Cm[0, :, 0], st) + D[h] * x[0, :, h]
        assert rel(y[0, :, h], yy) < 1e-12
        assert rel(f[0, h], st[-1]) < 1e-12


@pytest.mark.parametrize("Q", [1, 4, 16, 19])
def test_input_dt_chunked_equals_recurrence(Q):
    p = rand_problem(seed=13, Bz=2, L=37, H=4, P=2, N=3, G=2)
    y, f = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], input_dt=True)
    out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], Q, p["D"], p["init"], input_dt=True)
    assert rel(out["y"], y) < 1e-12 and rel(out["final"], f) < 1e-12
