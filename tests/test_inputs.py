"""The seeded input generator (CPU only)."""
import math

import numpy as np
import pytest

from chunked_state_space_b200 import inputs

MASK = (1 << 64) - 1


def _splitmix64_py(state, n):
    """splitmix64 as published (Steele, Lea, Flood 2014), in Python integers."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_stream():
    # the first output of splitmix64 from state 0 is the widely quoted 0xE220A8397B1DCDAF
    assert int(inputs.raw_u64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF
    key = inputs.stream_key(0, 2, 0, "x")
    got = [int(v) for v in inputs.raw_u64(key, 0, 16)]
    assert got == _splitmix64_py(key, 16)
    # counter-based: a slice regenerates on its own
    assert [int(v) for v in inputs.raw_u64(key, 5, 3)] == got[5:8]


def test_fill_slices_and_determinism():
    key = inputs.stream_key(0, 1, 0, "x")
    full = inputs.fill((1000,), "f32", key, inputs.NORMAL, 0.0, 1.0)
    part = inputs.fill((100,), "f32", key, inputs.NORMAL, 0.0, 1.0, first=450)
    np.testing.assert_array_equal(full[450:550], part)
    np.testing.assert_array_equal(full, inputs.fill((1000,), "f32", key, inputs.NORMAL, 0.0, 1.0))


def test_bf16_output_is_rne_of_fp32():
    torch = pytest.importorskip("torch")
    key = inputs.stream_key(0, 3, 0, "B")
    f = inputs.fill((4096,), "f32", key, inputs.NORMAL, 0.0, 0.1)
    b = inputs.fill((4096,), "bf16", key, inputs.NORMAL, 0.0, 0.1)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(b, ref)


def test_distributions():
    wl = inputs.custom("mamba2_2p7b_layer", batch=1, seqlen=2048)
    t = inputs.generate(wl)
    x = t["x"]
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    assert abs(xf.mean()) < 0.01 and abs(xf.std() - 1.0) < 0.01
    assert t["dt"].min() > 0 and abs(np.mean(np.log(np.expm1(t["dt"].astype(np.float64)))) + 2.0) < 0.02
    assert np.all(t["A"] <= -1.0) and np.all(t["A"] >= -16.0)
    bf = inputs.bf16_bits_to_f32(t["B"]).astype(np.float64)
    assert abs(bf.std() - 1 / math.sqrt(128)) < 0.002
    init = t["init"].astype(np.float64)
    assert abs(init.var() - 0.1) < 0.005
    tiny = inputs.generate(inputs.WORKLOADS["tiny_f32"])
    assert np.all(tiny["D"] == 0) and np.all(tiny["init"] == 0) and tiny["x"].dtype == np.float32
    assert inputs.generate(inputs.WORKLOADS["long_context_layer"], names=("A",))["A"].shape == (80,)


def test_streams_differ_by_tensor_layer_and_workload():
    keys = {inputs.stream_key(0, w, l, n) for w in range(5) for l in range(3) for n in inputs.TENSOR_IDS}
    assert len(keys) == 5 * 3 * len(inputs.TENSOR_IDS)
