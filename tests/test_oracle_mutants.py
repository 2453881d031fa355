"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case copies oracle/ssd_oracle.c, plants one plausible mistake (a dropped
term, a wrong index, a transposed operand, an off-by-one in a decay product),
compiles the copy into a temporary library and runs the pin checks of
tests/test_oracle.py against it.  A mutant that passes every pin would mean
the pins cannot see that kind of error.
"""
import math
import os

import numpy as np
import pytest

import oracle
from test_oracle import _read_golden, brute_force, rand_problem, rel
import test_oracle_vdecay as vd

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ssd_oracle.c")

MUTANTS = {
    "decay_dropped": ("row[p] = a * row[p] + u * bn * xt[p];", "row[p] = row[p] + u * bn * xt[p];"),
    "input_dt_factor_dropped": ("const double u = input_dt ? dt[(b * L + t) * H + h] : 1.0;", "const double u = 1.0;"),
    "input_dt_chunked_intra_dropped": ("const double w = cb * Lts * (input_dt ? dt[(b * L + s) * H + h] : 1.0);",
                                       "const double w = cb * Lts;"),
    "input_dt_chunked_state_dropped": ("if (input_dt) w *= dt[(b * L + s) * H + h];", ""),
    "group_index": ("const int64_t b = bh / H, h = bh % H, g = h / hpg;",
                    "const int64_t b = bh / H, h = bh % H, g = h % G;"),
    "b_c_swapped": ("const double bn = bt[n];", "const double bn = ct[n];"),
    "skip_dropped": ("yt[p] = d * xt[p];", "yt[p] = 0.0 * xt[p];"),
    "decay_sign": ("const double a = exp(dt[(b * L + t) * H + h] * A[h]);",
                   "const double a = exp(-dt[(b * L + t) * H + h] * A[h]);"),
    "state_transposed": ("for (int64_t p = 0; p < P; ++p) yt[p] += cn * row[p];",
                         "for (int64_t p = 0; p < P; ++p) yt[p] += cn * st[(p * N + n) % (N * P)];"),
    "inter_exclusive": ("for (int64_t j = 0; j <= i; ++j) dl *= a[j];",
                        "for (int64_t j = 0; j < i; ++j) dl *= a[j];"),
    "intra_mask_shift": ("if (j < i) Lts *= a[j + 1];", "if (j < i) Lts *= a[j];"),
    "state_weight_shift": ("for (int64_t r = j + 1; r < len; ++r) w *= a[r];",
                           "for (int64_t r = j; r < len; ++r) w *= a[r];"),
    "recursion_decay_dropped": ("prev[k] = bin[k] + Ac * prev[k];", "prev[k] = bin[k] + prev[k];"),
    "lam_missing_A": ("if (i < len) s += dt[(b * L + c0 + i) * H + h] * A[h];",
                      "if (i < len) s += dt[(b * L + c0 + i) * H + h];"),
    "rms_count": ("ss / (double)F", "ss / (double)(F - 1)"),
    "rms_eps_dropped": ("const double inv = 1.0 / sqrt(ss / (double)F + eps);",
                        "const double inv = 1.0 / sqrt(ss / (double)F);"),
    "vdecay_channel_reversed": ("const double a = exp(dtv * Av[h * N + n]);",
                                "const double a = exp(dtv * Av[h * N + (N - 1 - n)]);"),
    "vdecay_decay_dropped": ("for (int64_t p = 0; p < P; ++p) row[p] = a * row[p] + bt[n] * xt[p];",
                             "for (int64_t p = 0; p < P; ++p) row[p] = row[p] + bt[n] * xt[p];"),
    "vdecay_chunked_mask_shift": ("for (int64_t n = 0; n < N; ++n) w[n] *= a[(j + 1) * N + n];",
                                  "for (int64_t n = 0; n < N; ++n) w[n] *= a[j * N + n];"),
    "vdecay_chunked_inter_exclusive": ("for (int64_t j = 0; j <= i; ++j) dl *= a[j * N + n];",
                                       "for (int64_t j = 0; j < i; ++j) dl *= a[j * N + n];"),
    "vdecay_chunked_state_weight_shift": ("for (int64_t r = j + 1; r < len; ++r) wn *= a[r * N + n];",
                                          "for (int64_t r = j; r < len; ++r) wn *= a[r * N + n];"),
    "vdecay_recursion_decay_dropped": ("prev[n * P + p] = bin[n * P + p] + Ac * prev[n * P + p];",
                                       "prev[n * P + p] = bin[n * P + p] + prev[n * P + p];"),
    "bf16_truncates": ("nearbyint(ldexp(m, 8))", "trunc(ldexp(m, 8))"),
}


def _pins(o):
    """Run the pins against oracle handle `o`; return the names of those that fail."""
    failed = []

    def check(name, fn):
        try:
            with np.errstate(all="ignore"):
                ok = bool(fn())
        except Exception:
            ok = False
        if not ok:
            failed.append(name)

    g = _read_golden("scalar_recurrence.txt")
    L = len(g["dt"])
    args = (g["x"].reshape(1, L, 1, 1), g["dt"].reshape(1, L, 1), g["A"], g["B"].reshape(1, L, 1, 1),
            g["C"].reshape(1, L, 1, 1), g["D"], g["h0"].reshape(1, 1, 1, 1))

    def golden():
        y, f = oracle.scan_recurrence(*args, o=o)
        return np.allclose(y.ravel(), g["y"], atol=1e-12) and np.allclose(f.ravel(), g["final"], atol=1e-12)
    check("golden", golden)

    p = rand_problem(seed=4, Bz=2, L=17, H=4, P=2, N=3, G=2)

    def brute():
        y, f = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], o=o)
        yb, fb = brute_force(p)
        return rel(y, yb) < 1e-12 and rel(f, fb) < 1e-12
    check("brute_force", brute)

    def chunked():
        y, f = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], o=o)
        for Q in (1, 4, 16):
            out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], Q, p["D"], p["init"], o=o)
            if not (rel(out["y"], y) < 1e-12 and rel(out["final"], f) < 1e-12):
                return False
        return True
    check("chunked_vs_recurrence", chunked)

    def input_dt_brute():
        y, f = oracle.scan_recurrence(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], p["D"], p["init"], o=o,
                                      input_dt=True)
        yb, fb = brute_force(p, input_dt=True)
        return rel(y, yb) < 1e-12 and rel(f, fb) < 1e-12
    check("input_dt_brute_force", input_dt_brute)

    def input_dt_chunked():
        yb, fb = brute_force(p, input_dt=True)
        for Q in (4, 16):
            out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], Q, p["D"], p["init"], o=o,
                                      input_dt=True)
            if not (rel(out["y"], yb) < 1e-12 and rel(out["final"], fb) < 1e-12):
                return False
        return True
    check("input_dt_chunked", input_dt_chunked)

    gd = _read_golden("scalar_recurrence_input_dt.txt")

    def golden_input_dt():
        Ld = len(gd["dt"])
        y, f = oracle.scan_recurrence(gd["x"].reshape(1, Ld, 1, 1), gd["dt"].reshape(1, Ld, 1), gd["A"],
                                      gd["B"].reshape(1, Ld, 1, 1), gd["C"].reshape(1, Ld, 1, 1), gd["D"],
                                      gd["h0"].reshape(1, 1, 1, 1), o=o, input_dt=True)
        return np.allclose(y.ravel(), gd["y"], atol=1e-12) and np.allclose(f.ravel(), gd["final"], atol=1e-12)
    check("golden_input_dt", golden_input_dt)

    def lam():
        out = oracle.scan_chunked(p["x"], p["dt"], p["A"], p["Bm"], p["Cm"], 5, p["D"], p["init"], o=o)
        a = np.exp(p["dt"][0, :5, 0] * p["A"][0])
        return np.allclose(np.exp(out["lam"][0, 0, 0]), np.cumprod(a), rtol=1e-12)
    check("lam", lam)

    def rms():
        a = np.zeros((1, 1, 3, 4))
        a[0, 0, 1, 2] = -7.5
        out = oracle.rmsnorm_bf16(a, 0.0, o=o)
        return out[0, 0, 1, 2] == -3.46875  # bf16(-sqrt(12)) worked by hand: sqrt(12) = 3.4641...
    check("rmsnorm_one_hot", rms)

    def rms_eps():
        a = np.zeros((1, 1, 3, 4))
        a[0, 0, 1, 2] = -7.5
        out = oracle.rmsnorm(a, 0.25, o=o)
        return abs(out[0, 0, 1, 2] - (-7.5 / math.sqrt(4.9375))) < 1e-15  # 56.25 / 12 + 0.25 = 4.9375
    check("rmsnorm_eps", rms_eps)

    gv = vd._read_golden("vector_decay.txt")

    def golden_vdecay():
        Lv, Nv = 3, 2
        args_v = (gv["x"].reshape(1, Lv, 1, 1), gv["dt"].reshape(1, Lv, 1), gv["Av"].reshape(1, Nv),
                  gv["B"].reshape(1, Lv, 1, Nv), gv["C"].reshape(1, Lv, 1, Nv))
        y, f = oracle.scan_recurrence_vdecay(*args_v, gv["D"], gv["h0"].reshape(1, 1, Nv, 1), o=o)
        return np.allclose(y.ravel(), gv["y"], atol=1e-12) and np.allclose(f.ravel(), gv["final"], atol=1e-12)
    check("golden_vdecay", golden_vdecay)

    pv = vd.problem(Bz=1, L=17, H=2, P=2, N=3, G=1, seed=5)

    def vdecay_chunked():
        y, f = oracle.scan_recurrence_vdecay(*pv, o=o)
        for Q in (1, 4, 16):
            yc, fc = oracle.scan_chunked_vdecay(*pv[:5], Q, pv[5], pv[6], o=o)
            if not (rel(yc, y) < 1e-12 and rel(fc, f) < 1e-12):
                return False
        return True
    check("vdecay_chunked_vs_recurrence", vdecay_chunked)

    def vdecay_golden_chunked():
        Lv, Nv = 3, 2
        args_v = (gv["x"].reshape(1, Lv, 1, 1), gv["dt"].reshape(1, Lv, 1), gv["Av"].reshape(1, Nv),
                  gv["B"].reshape(1, Lv, 1, Nv), gv["C"].reshape(1, Lv, 1, Nv))
        for Q in (2, 3):
            y, f = oracle.scan_chunked_vdecay(*args_v, Q, gv["D"], gv["h0"].reshape(1, 1, Nv, 1), o=o)
            if not (np.allclose(y.ravel(), gv["y"], atol=1e-12) and np.allclose(f.ravel(), gv["final"], atol=1e-12)):
                return False
        return True
    check("vdecay_golden_chunked", vdecay_golden_chunked)

    def bf16():
        v = np.array([1.0 + 3 * 2.0 ** -9, -(1.0 + 2.0 ** -8 + 2.0 ** -10)])
        # nearest bf16 values worked by hand: 1 + 2^-7 and -(1 + 2^-7)
        return np.array_equal(oracle.round_bf16(v, o=o), np.array([1.0 + 2.0 ** -7, -(1.0 + 2.0 ** -7)]))
    check("bf16_rounding", bf16)
    return failed


def test_pins_pass_on_real_oracle():
    assert _pins(oracle.load()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mut.c"
    path.write_text(mutated)
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / "libmut.so"))
    o = oracle.load(lib)
    assert _pins(o) != [], f"mutant {name} passed every pin"
