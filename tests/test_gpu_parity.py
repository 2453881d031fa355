"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (max|y - y_ref| / max|y_ref|, same for the final state):
1e-5 for fp32 io, 5e-3 for bf16 io with fp32 accumulation.
"""
import numpy as np
import pytest
import torch

import oracle
from chunked_state_space_b200 import inputs
from chunked_state_space_b200 import ssd
from gpu_util import TOL, device_inputs, oracle_args, oracle_sampled, rel_err, to_dev, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ssd.lib()  # fails loudly if libssd.so is missing
    yield
    torch.cuda.synchronize()


def run_scan(dev, wl, unfused=False, **kw):
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, unfused=unfused, **kw)
    torch.cuda.synchronize()
    return y, fin


def check_full(wl, seed=0, paths=("default", "unfused")):
    host = inputs.generate(wl, seed=seed)
    dev = device_inputs(host)
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host))
    for path in paths:
        y, fin = run_scan(dev, wl, unfused=(path == "unfused"))
        ey, ef = rel_err(to_np64(y), y_ref), rel_err(to_np64(fin), f_ref)
        assert ey <= TOL[wl.io], (path, ey)
        assert ef <= TOL[wl.io], (path, ef)
    return host, dev


# ------------------------------------------------------------------ small workloads, whole output

def test_tiny_f32_workload():
    check_full(inputs.WORKLOADS["tiny_f32"])


@pytest.mark.parametrize("over", [
    dict(base="tiny_f32", batch=2, seqlen=300, nheads=4, ngroups=2, headdim=16, dstate=16, chunk=64),
    dict(base="tiny_f32", batch=1, seqlen=1, nheads=2, chunk=64),
    dict(base="tiny_f32", batch=1, seqlen=50, nheads=2, chunk=64),         # L < Q
    dict(base="tiny_f32", batch=2, seqlen=33, nheads=3, ngroups=3, headdim=5, dstate=3, chunk=1),
    dict(base="tiny_f32", batch=1, seqlen=130, nheads=2, headdim=1, dstate=1, chunk=16),
    dict(base="tiny_f32", batch=1, seqlen=517, nheads=2, headdim=64, dstate=128, chunk=256, init_var=0.5),
    dict(base="mamba2_130m_layer", batch=2, seqlen=700, nheads=4, ngroups=2, init_var=0.1),
    dict(base="mamba2_130m_layer", batch=1, seqlen=1, nheads=2),
    dict(base="mamba2_130m_layer", batch=1, seqlen=255, nheads=2, init_var=0.1),
    dict(base="mamba2_130m_layer", batch=1, seqlen=1000, nheads=3, headdim=32, dstate=64, chunk=128),
    dict(base="mamba2_130m_layer", batch=1, seqlen=200, nheads=2, headdim=7, dstate=9, chunk=40),
])
def test_shapes_and_edges(over):
    over = dict(over)
    base = over.pop("base")
    check_full(inputs.custom(base, **over))


def test_no_d_no_init_and_aliasing():
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=600, nheads=2, init_var=0.1)
    host = inputs.generate(wl)
    dev = device_inputs(host)
    args = oracle_args(host)
    y_ref, f_ref = oracle.scan_recurrence(*args[:5], None, None)
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], None, None, chunk=wl.chunk)
    torch.cuda.synchronize()
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(fin), f_ref) <= TOL["bf16"]
    # final_state may alias init_state
    y_ref2, f_ref2 = oracle.scan_recurrence(*args)
    st = dev["init"].clone()
    y2, _ = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], st, chunk=wl.chunk,
                             final_state=st)
    torch.cuda.synchronize()
    assert rel_err(to_np64(y2), y_ref2) <= TOL["bf16"]
    assert rel_err(to_np64(st), f_ref2) <= TOL["bf16"]


def test_deterministic():
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=1100, nheads=4, init_var=0.1)
    dev = device_inputs(inputs.generate(wl))
    y1, f1 = run_scan(dev, wl)
    y2, f2 = run_scan(dev, wl)
    assert torch.equal(y1, y2) and torch.equal(f1, f2)


# ------------------------------------------------------------------ decay extremes on the tensor-core path

def _decay_regime(host, regime):
    L, H = host["dt"].shape[1], host["dt"].shape[2]
    if regime == "A_zero":            # a == 1: no decay at all, the state is a prefix sum
        host["A"][:] = 0.0
    elif regime == "dt_zero":         # a == 1 through dt = 0 (the input term stays)
        host["dt"][:] = 0.0
    elif regime == "strong":          # dt*A = -64 per token: every past token is forgotten
        host["A"][:] = -16.0
        host["dt"][:] = 4.0
    elif regime == "mixed":           # long undecayed runs cut by abrupt strong decay, per head
        host["A"][:] = np.array([0.0, -16.0, -1.0, -0.01] * (H // 4 + 1), dtype=np.float32)[:H]
        t = np.arange(L)
        host["dt"][:] = np.where((t // 37) % 3 == 0, 4.0, 1e-3).astype(np.float32)[None, :, None]
    return host


@pytest.mark.parametrize("regime", ["A_zero", "dt_zero", "strong", "mixed"])
@pytest.mark.parametrize("input_dt", [False, True])
@pytest.mark.parametrize("two_heads", [False, True])
def test_fused_decay_extremes(regime, input_dt, two_heads):
    """Both fused tensor-core kernels at the ends of the decay range, against the
    oracle: a == 1 over whole 128-token sub-chunks (the off-diagonal factors stay
    1), and |dt*A| = 64 per token (every factor below the diagonal underflows to
    zero; only the diagonal terms survive), and both mixed within one sequence."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=700, nheads=4, ngroups=2, init_var=0.1)
    host = _decay_regime(inputs.generate(wl), regime)
    dev = device_inputs(host)
    path = ssd.ssd_scan_path(ssd.make_dims(dev["x"], dev["B"], wl.chunk, input_dt, two_heads))[0]
    assert path == ("fused_pair" if two_heads else "fused")
    y, fin = ssd.ssd_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init"],
                              chunk=wl.chunk, input_dt=input_dt, two_heads=two_heads)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.scan_recurrence(*oracle_args(host), input_dt=input_dt)
    ey, ef = rel_err(to_np64(y), y_ref), rel_err(to_np64(fin), f_ref)
    assert ey <= TOL["bf16"], ey
    assert ef <= TOL["bf16"], ef
    assert torch.isfinite(y.float()).all() and torch.isfinite(fin).all()


# ------------------------------------------------------------------ the four steps, one at a time

@pytest.mark.parametrize("case", ["f32", "bf16_tensor_cores", "bf16_cuda_cores"])
def test_steps_match_oracle_intermediates(case):
    """Each step kernel on the oracle's inputs to that step.  bf16 with P = 64,
    N = 128, Q % 128 = 0 runs steps 2 and 4 on tcgen05; other bf16 shapes on
    CUDA cores."""
    if case == "f32":
        wl = inputs.custom("tiny_f32", batch=2, seqlen=300, nheads=4, ngroups=2, init_var=0.3)
    elif case == "bf16_tensor_cores":
        wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=700, nheads=4, ngroups=2, init_var=0.1)
    else:
        wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=700, nheads=4, ngroups=2, headdim=32, dstate=64,
                           chunk=128, init_var=0.1)
    io = wl.io
    tol = TOL[io]
    host = inputs.generate(wl)
    dev = device_inputs(host)
    args = oracle_args(host)
    ref = oracle.scan_chunked(*args[:5], wl.chunk, args[5], args[6])
    x, Bm = dev["x"], dev["B"]
    dims = ssd.make_dims(x, Bm, wl.chunk)
    f32 = lambda a: torch.from_numpy(a.astype(np.float32)).cuda()
    # step 1
    lam = ssd.ssd_chunk_cumsum(dev["dt"], dev["A"], dims)
    torch.cuda.synchronize()
    assert rel_err(to_np64(lam), ref["lam"]) <= 1e-6
    # step 2 on the oracle's lam
    cs = ssd.ssd_chunk_state(x, Bm, f32(ref["lam"]), dims)
    torch.cuda.synchronize()
    assert rel_err(to_np64(cs), ref["chunk_states"]) <= tol
    # step 3 on the oracle's chunk states
    prev, fin = ssd.ssd_state_passing(f32(ref["chunk_states"]), f32(ref["lam"]), dims, init_state=dev["init"])
    torch.cuda.synchronize()
    assert rel_err(to_np64(prev), ref["prev_states"]) <= 1e-5
    assert rel_err(to_np64(fin), ref["final"]) <= 1e-5
    # step 3 in place (prev aliases chunk states)
    buf = f32(ref["chunk_states"])
    ssd.ssd_state_passing(buf, f32(ref["lam"]), dims, init_state=dev["init"], prev_states=buf)
    torch.cuda.synchronize()
    assert rel_err(to_np64(buf), ref["prev_states"]) <= 1e-5
    # step 4 on the oracle's prev states
    y = ssd.ssd_chunk_scan(x, Bm, dev["C"], f32(ref["lam"]), f32(ref["prev_states"]), dims, D=dev["D"])
    torch.cuda.synchronize()
    assert rel_err(to_np64(y), ref["y"]) <= tol


@pytest.mark.parametrize("chunk,cpc", [(256, 2), (256, 3), (128, 4), (128, 16)])
def test_step_kernels_with_several_chunks_per_cta(chunk, cpc):
    """Steps 2 and 4 on tcgen05 with cpc consecutive chunks of a sequence per
    CTA (the chunk-scan kernel takes the next chunk's given state at each chunk
    boundary): 1700 tokens give 7 or 14 chunks, so the last CTA of a sequence
    holds fewer chunks and a ragged last chunk; the unfused scan runs the same
    kernels end to end."""
    wl = inputs.custom("mamba2_130m_layer", batch=2, seqlen=1700, nheads=3, ngroups=1, chunk=chunk,
                       init_var=0.1)
    tol = TOL[wl.io]
    host = inputs.generate(wl, seed=5)
    dev = device_inputs(host)
    args = oracle_args(host)
    ref = oracle.scan_chunked(*args[:5], wl.chunk, args[5], args[6])
    x, Bm = dev["x"], dev["B"]
    dims = ssd.make_dims(x, Bm, wl.chunk)
    f32 = lambda a: torch.from_numpy(a.astype(np.float32)).cuda()
    ssd.ssd_selftest_set_step_chunks(cpc)
    try:
        cs = ssd.ssd_chunk_state(x, Bm, f32(ref["lam"]), dims)
        y = ssd.ssd_chunk_scan(x, Bm, dev["C"], f32(ref["lam"]), f32(ref["prev_states"]), dims, D=dev["D"])
        y2, fin2 = run_scan(dev, wl, unfused=True)
    finally:
        ssd.ssd_selftest_set_step_chunks(0)
    torch.cuda.synchronize()
    assert rel_err(to_np64(cs), ref["chunk_states"]) <= tol
    assert rel_err(to_np64(y), ref["y"]) <= tol
    assert rel_err(to_np64(y2), ref["y"]) <= tol
    assert rel_err(to_np64(fin2), ref["final"]) <= tol
    # the chosen split gives the same chunk states to the fp32 rounding of the tiles
    cs0 = ssd.ssd_chunk_state(x, Bm, f32(ref["lam"]), dims)
    torch.cuda.synchronize()
    assert rel_err(to_np64(cs0), to_np64(cs)) <= 1e-5


@pytest.mark.parametrize("shape,dtype", [
    ((2, 37, 24, 64), torch.bfloat16),   # 74 rows (not a multiple of 8), 16-byte vectors
    ((1, 5, 3, 5), torch.bfloat16),      # 15 features: the scalar path
    ((2, 9, 4, 16), torch.float32),
])
def test_rmsnorm_matches_oracle(shape, dtype):
    rng = np.random.default_rng(0)
    a = rng.standard_normal(shape).astype(np.float32) * 3.0
    t = torch.from_numpy(a).cuda().to(dtype)
    out = ssd.ssd_rmsnorm(t, 1e-6)
    torch.cuda.synchronize()
    if dtype == torch.bfloat16:
        ref = oracle.rmsnorm_bf16(to_np64(t), 1e-6)
        # both round to bf16: compare within one bf16 ulp of the normalised values
        assert np.max(np.abs(to_np64(out) - ref)) <= 2.0 ** -7 * np.max(np.abs(ref))
    else:
        ref = oracle.rmsnorm(to_np64(t), 1e-6)
        assert np.max(np.abs(to_np64(out) - ref)) <= 1e-5 * np.max(np.abs(ref))
    # in place
    t2 = t.clone()
    ssd.ssd_rmsnorm(t2, 1e-6, out=t2)
    torch.cuda.synchronize()
    assert torch.equal(t2, out)


# ------------------------------------------------------------------ the named workloads at full size

def test_mamba2_130m_layer_full():
    check_full(inputs.WORKLOADS["mamba2_130m_layer"])


def _sample_pairs(Bz, H, n, seed):
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (Bz - 1, H - 1)}
    while len(pairs) < n:
        pairs.add((int(rng.integers(Bz)), int(rng.integers(H))))
    return sorted(pairs)


@pytest.mark.slow
@pytest.mark.parametrize("name,nsamp", [("mamba2_2p7b_layer", 12), ("long_context_layer", 6)])
def test_full_size_sampled(name, nsamp):
    """Full-size run in the benchmark's launch configuration.  The oracle checks
    (1) sampled (batch, head) rows over the whole sequence and their final
    states, and (2) the whole output tensor -- every batch and head -- over the
    first 2048 tokens (y is causal, so the prefix of the full run is the run of
    the prefix)."""
    wl = inputs.WORKLOADS[name]
    host = inputs.generate(wl)
    dev = device_inputs(host)
    y, fin = run_scan(dev, wl)
    pairs = _sample_pairs(wl.batch, wl.nheads, nsamp, seed=1)
    y_ref, f_ref = oracle_sampled(host, wl, pairs)
    for i, (b, h) in enumerate(pairs):
        ey = rel_err(to_np64(y[b, :, h]), y_ref[i])
        ef = rel_err(to_np64(fin[b, h]), f_ref[i])
        assert ey <= TOL["bf16"], (b, h, ey)
        assert ef <= TOL["bf16"], (b, h, ef)
    assert torch.isfinite(y.float()).all()
    del y_ref, f_ref
    Lp = 2048
    f = inputs.to_f64
    pre = {k: f(host[k][:, :Lp]) for k in ("x", "dt", "B", "C")}
    y_pre, _ = oracle.scan_recurrence(pre["x"], pre["dt"], f(host["A"]), pre["B"], pre["C"], f(host["D"]),
                                      f(host["init"]))
    got = to_np64(y[:, :Lp])
    e_all = rel_err(got, y_pre)
    # per (batch, head) normalised by that sequence's own max: reported, not
    # asserted (the parity metric normalises by the tensor's max)
    per = np.max(np.abs(got - y_pre), axis=(1, 3)) / np.maximum(np.max(np.abs(y_pre), axis=(1, 3)), 1e-30)
    print(f"{name}: whole tensor, first {Lp} tokens: rel err {e_all:.3e}, worst (b, h) own-max {per.max():.3e}")
    assert e_all <= TOL["bf16"], e_all
    del dev, y, fin
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ multi-layer stack: vertical vs horizontal

def _stack_layers(wl, n_layers):
    layers_host = [inputs.generate(wl, layer=l, names=("dt", "A", "B", "C", "D")) for l in range(n_layers)]
    return layers_host, [device_inputs(h) for h in layers_host]


def _horizontal_normed(x0, layers, states, wl, eps):
    """The layer-major schedule through the public one-layer call with the norm
    fused (ssd_scan_fwd_normed): every layer's y and the sums of squares it
    passes on.  Returns (ys, sums) with sums[l] the input sums of layer l."""
    ys, sums = [], [None]
    x = x0
    for l, p in enumerate(layers):
        y, ss, _ = ssd.ssd_scan_fwd_normed(x, sums[-1], p["dt"], p["A"], p["B"], p["C"], p["D"], states[l],
                                           chunk=wl.chunk, rms_eps=eps, final_state=states[l],
                                           want_sums=l + 1 < len(layers))
        ys.append(y)
        sums.append(ss)
        x = y
    torch.cuda.synchronize()
    return ys, sums[:-1]


def _normed_input(y_prev, eps, b, h, tok_block=4096):
    """The input layer l+1 sees, for batch b and head h: the previous layer's
    stored y RMS-normalised over each token's H*P features (oracle.rmsnorm,
    fp64, unrounded: the fused path never stores it), in token blocks."""
    L = y_prev.shape[1]
    out = np.empty((L, y_prev.shape[3]))
    for t0 in range(0, L, tok_block):
        out[t0:t0 + tok_block] = oracle.rmsnorm(to_np64(y_prev[b:b + 1, t0:t0 + tok_block]), eps)[0, :, h]
    return out


@pytest.mark.parametrize("L,V", [(1024, 256), (1000, 256), (1000, 300)])
def test_vertical_small(L, V):
    """3-layer stack with the RMS norm fused between layers: vertical ==
    horizontal (bitwise when V % Q == 0), every layer teacher-forced against
    the oracle on its own input (the previous GPU layer's y, normalised by the
    oracle; 5e-3), the sums of squares each layer passes on, and the end-to-end
    output within the bound of _check_end_to_end."""
    wl = inputs.custom("stack24_vertical", batch=2, seqlen=L, nheads=4)
    n_layers, eps = 3, 1e-6
    host_layers, dev_layers = _stack_layers(wl, n_layers)
    x0h = inputs.generate(wl, names=("x",))["x"]
    x0 = to_dev(x0h)
    zero = lambda: [torch.zeros((wl.batch, wl.nheads, wl.dstate, wl.headdim), device="cuda")
                    for _ in range(n_layers)]
    st_v, st_h = zero(), zero()
    yv = ssd.ssd_vertical_fwd(x0, dev_layers, st_v, vblock=V, chunk=wl.chunk, rms_eps=eps)
    ys, sums = _horizontal_normed(x0, dev_layers, st_h, wl, eps)
    if V % wl.chunk == 0:
        assert torch.equal(yv, ys[-1])
        for a, b in zip(st_v, st_h):
            assert torch.equal(a, b)
    f = inputs.to_f64
    layers64 = [dict(dt=f(h["dt"]), A=f(h["A"]), B=f(h["B"]), C=f(h["C"]), D=f(h["D"])) for h in host_layers]
    for l, p in enumerate(layers64):
        x_in = f(x0h) if l == 0 else oracle.rmsnorm(to_np64(ys[l - 1]), eps)
        y_ref, f_ref = oracle.scan_recurrence(x_in, p["dt"], p["A"], p["B"], p["C"], p["D"], None)
        assert rel_err(to_np64(ys[l]), y_ref) <= TOL["bf16"], ("layer", l)
        assert rel_err(to_np64(st_h[l]), f_ref) <= TOL["bf16"], ("state", l)
        assert rel_err(to_np64(st_v[l]), f_ref) <= TOL["bf16"], ("vertical state", l)
        if l > 0:  # the sums layer l read: over the P values of the stored y_{l-1}
            ss_ref = np.sum(to_np64(ys[l - 1]) ** 2, axis=-1)
            assert rel_err(to_np64(sums[l]), ss_ref) <= 1e-5, ("sums", l)
    _check_end_to_end(f(x0h), layers64, eps, to_np64(yv), tag=f"3-layer stack L={L} V={V}")


@pytest.mark.parametrize("nheads,seqlen", [(6, 1000), (36, 300)])
def test_normed_scan_chains_two_layers(nheads, seqlen):
    """ssd_scan_fwd_normed on head counts that are not a multiple of 4 (the
    scalar sums path) and above 32 (sums past the prefetched first 32 heads),
    with a ragged sequence: layer 1's y against the oracle on the input it sees
    (layer 0's stored y, normalised by the oracle), and the sums layer 0 passes
    on against those of its stored y."""
    wl = inputs.custom("stack24_vertical", batch=2, seqlen=seqlen, nheads=nheads, ngroups=2)
    host_layers, dev_layers = _stack_layers(wl, 2)
    x0h = inputs.generate(wl, names=("x",))["x"]
    x0 = to_dev(x0h)
    states = [torch.zeros((wl.batch, wl.nheads, wl.dstate, wl.headdim), device="cuda") for _ in range(2)]
    eps = 1e-6
    ys, sums = _horizontal_normed(x0, dev_layers, states, wl, eps)
    np.testing.assert_allclose(to_np64(sums[1]), np.sum(to_np64(ys[0]) ** 2, axis=-1), rtol=1e-5, atol=0)
    f = inputs.to_f64
    h = host_layers[1]
    y_ref, f_ref = oracle.scan_recurrence(oracle.rmsnorm(to_np64(ys[0]), eps), f(h["dt"]), f(h["A"]), f(h["B"]),
                                          f(h["C"]), f(h["D"]), None)
    assert rel_err(to_np64(ys[1]), y_ref) <= TOL["bf16"]
    assert rel_err(to_np64(states[1]), f_ref) <= TOL["bf16"]


def test_vertical_two_heads_keeps_the_norm_pass():
    """With two heads per CTA the stack keeps the norm as its own pass
    (ssd_rmsnorm between layers, the normalised input stored in bf16): vertical
    == that horizontal schedule bitwise, and the last layer teacher-forced
    against the oracle on the stored input."""
    wl = inputs.custom("stack24_vertical", batch=2, seqlen=1024, nheads=4)
    n_layers, eps, V = 3, 1e-6, 256
    host_layers, dev_layers = _stack_layers(wl, n_layers)
    x0 = to_dev(inputs.generate(wl, names=("x",))["x"])
    zero = lambda: [torch.zeros((wl.batch, wl.nheads, wl.dstate, wl.headdim), device="cuda")
                    for _ in range(n_layers)]
    st_v, st_h = zero(), zero()
    yv = ssd.ssd_vertical_fwd(x0, dev_layers, st_v, vblock=V, chunk=wl.chunk, rms_eps=eps, two_heads=True)
    xs, y = [x0], None
    for l, p in enumerate(dev_layers):
        y, _ = ssd.ssd_scan_fwd(xs[-1], p["dt"], p["A"], p["B"], p["C"], p["D"], st_h[l], chunk=wl.chunk,
                                final_state=st_h[l], two_heads=True)
        if l + 1 < n_layers:
            xs.append(ssd.ssd_rmsnorm(y, eps))
    torch.cuda.synchronize()
    assert torch.equal(yv, y)
    for a, b in zip(st_v, st_h):
        assert torch.equal(a, b)
    f = inputs.to_f64
    h = host_layers[-1]
    y_ref, _ = oracle.scan_recurrence(to_np64(xs[-1]), f(h["dt"]), f(h["A"]), f(h["B"]), f(h["C"]), f(h["D"]), None)
    assert rel_err(to_np64(y), y_ref) <= TOL["bf16"]


def _check_end_to_end(x0, layers64, eps, y_end, tag="stack"):
    """End-to-end comparison of a GPU layer stack with the oracle's stack.

    Every GPU layer is checked on its own (teacher-forced, 5e-3) elsewhere; the
    whole stack also carries each layer's error into the layers after it.  The
    bound models a correct bf16 implementation: each layer's output deviates
    from the exact map by about one bf16 rounding per element (the kernel
    multiplies bf16 operands P, X' and a bf16 copy of the state; the RMS
    relative error of one bf16 rounding is about 2^-9), and the oracle measures
    how far such independent per-layer noise moves its own last output (sens).
    Asserted: err <= 5e-3 + 2 * sens(2^-9).  The spread from rounding-boundary
    flips alone, sens(1e-7), is printed beside it: it leaves out the layers'
    compute errors, which every layer is allowed and which later layers
    amplify."""
    y_ref, _ = oracle.stack_horizontal(x0, layers64, eps)
    sens = rel_err(_stack_sensitivity(x0, layers64, eps, rel=2.0 ** -9), y_ref)
    flip = rel_err(_stack_sensitivity(x0, layers64, eps, rel=1e-7), y_ref)
    err = rel_err(y_end, y_ref)
    bound = TOL["bf16"] + 2.0 * sens
    print(f"{tag}: end-to-end err {err:.3e}, bound {bound:.3e} (sens(2^-9) {sens:.3e}; flips alone "
          f"sens(1e-7) {flip:.3e})")
    assert err <= bound, f"end-to-end err {err:.3e} > {bound:.3e} (sens {sens:.3e}, flips {flip:.3e})"


def _stack_sensitivity(x0, layers64, eps, rel, seed=0):
    """The oracle's own last-layer output when every layer's output is
    perturbed by independent relative noise of size `rel` (seeded Gaussian)
    before its bf16 storage rounding.  rel = 2^-9: about one bf16 rounding per
    element, the error a correct bf16 layer adds; rel = 1e-7: about one fp32
    rounding, which only changes which way values next to a bf16 rounding
    boundary round."""
    rng = np.random.default_rng(seed)
    x = x0
    y = None
    for li, p in enumerate(layers64):
        y, _ = oracle.scan_recurrence(x, p["dt"], p["A"], p["B"], p["C"], p["D"], None)
        if li + 1 < len(layers64):
            x = oracle.rmsnorm_bf16(oracle.round_bf16(y * (1 + rel * rng.standard_normal(y.shape))), eps)
    return y


@pytest.mark.slow
def test_stack24_vertical_full():
    """The 24-layer stack at full size (RMS norm fused between layers).

    1. vertical == horizontal bitwise on the GPU (V % Q == 0), the horizontal
       schedule run layer by layer through ssd_scan_fwd_normed;
    2. every layer, teacher-forced: the GPU's y_l and final state for a sampled
       (batch, head) over the whole sequence match the oracle run on the input
       the layer sees (y_{l-1} of the GPU, RMS-normalised by the oracle; 5e-3),
       and the sums of squares passed on are those of the stored y_l;
    3. end to end on a prefix against the oracle's stack, within the bound of
       _check_end_to_end.
    """
    wl = inputs.WORKLOADS["stack24_vertical"]
    n_layers, eps, V = wl.n_layers, 1e-6, wl.vblock
    host_layers, dev_layers = _stack_layers(wl, n_layers)
    x0h = inputs.generate(wl, names=("x",))["x"]
    x0 = to_dev(x0h)
    zero = lambda Bz: [torch.zeros((Bz, wl.nheads, wl.dstate, wl.headdim), device="cuda") for _ in range(n_layers)]
    st_v = zero(wl.batch)
    yv = ssd.ssd_vertical_fwd(x0, dev_layers, st_v, vblock=V, chunk=wl.chunk, rms_eps=eps)
    torch.cuda.synchronize()
    # horizontal schedule, keeping every layer's output and the sums it passes on
    st_h = zero(wl.batch)
    ys, sums = _horizontal_normed(x0, dev_layers, st_h, wl, eps)
    assert torch.equal(yv, ys[-1])
    for a, b in zip(st_v, st_h):
        assert torch.equal(a, b)
    # 2. teacher-forced per layer, one sampled (batch, head) per layer, full length, one oracle call
    rng = np.random.default_rng(2)
    samp = [(int(rng.integers(wl.batch)), int(rng.integers(wl.nheads))) for _ in range(n_layers)]
    f = inputs.to_f64
    xo = np.stack([to_np64(x0[b, :, h]) if l == 0 else _normed_input(ys[l - 1], eps, b, h)
                   for l, (b, h) in enumerate(samp)], axis=1)[None]
    dto = np.stack([f(host_layers[l]["dt"][b, :, h]) for l, (b, h) in enumerate(samp)], axis=1)[None]
    Bo = np.stack([f(host_layers[l]["B"][b, :, 0]) for l, (b, h) in enumerate(samp)], axis=1)[None]
    Co = np.stack([f(host_layers[l]["C"][b, :, 0]) for l, (b, h) in enumerate(samp)], axis=1)[None]
    Ao = np.array([f(host_layers[l]["A"])[h] for l, (b, h) in enumerate(samp)])
    Do = np.array([f(host_layers[l]["D"])[h] for l, (b, h) in enumerate(samp)])
    y_ref, f_ref = oracle.scan_recurrence(xo, dto, Ao, Bo, Co, Do, None)
    for l, (b, h) in enumerate(samp):
        assert rel_err(to_np64(ys[l][b, :, h]), y_ref[0, :, l]) <= TOL["bf16"], ("layer", l)
        assert rel_err(to_np64(st_h[l][b, h]), f_ref[0, l]) <= TOL["bf16"], ("state", l)
    for l in range(1, n_layers):
        tok = slice(0, 4096)
        ss_ref = np.sum(to_np64(ys[l - 1][:1, tok]) ** 2, axis=-1)
        assert rel_err(to_np64(sums[l][:1, tok]), ss_ref) <= 1e-5, ("sums", l)
    # 3. end to end on a prefix (batch 0, 1024 tokens); the prefix is causal, so
    # it equals the first 1024 tokens of the full run
    Lp = 1024
    pre = lambda t: t[:1, :Lp].contiguous()
    dev_pre = [dict(dt=pre(p["dt"]), A=p["A"], B=pre(p["B"]), C=pre(p["C"]), D=p["D"]) for p in dev_layers]
    yp = ssd.ssd_vertical_fwd(pre(x0), dev_pre, zero(1), vblock=V, chunk=wl.chunk, rms_eps=eps)
    torch.cuda.synchronize()
    assert torch.equal(yp, yv[:1, :Lp])
    layers64 = [dict(dt=f(h["dt"][:1, :Lp]), A=f(h["A"]), B=f(h["B"][:1, :Lp]), C=f(h["C"][:1, :Lp]),
                     D=f(h["D"])) for h in host_layers]
    _check_end_to_end(f(x0h[:1, :Lp]), layers64, eps, to_np64(yp), tag=f"stack24 (batch 0, {Lp} tokens)")
