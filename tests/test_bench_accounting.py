"""The roofline arithmetic of bench.py, on CPU.

The algorithmic bytes and flops per scan follow from the shapes alone: every
tensor the scan must read or write once (x, y, dt, B, C, A, D, the initial and
final states) and the causal contractions of the chunked form (C B^T shared by
the heads of a group, (S (.) L) X, the chunk state B^T X' and the inter-chunk
product C b).  These tests recompute them from the definitions for the
2.7B-shaped layer and check bench.py's helpers and its L2 rule.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from chunked_state_space_b200 import inputs  # noqa: E402


def test_algorithmic_bytes_of_the_2p7b_layer():
    wl = inputs.WORKLOADS["mamba2_2p7b_layer"]
    Bz, L, H, P, N, G = 8, 16384, 80, 64, 128, 1
    x = y = Bz * L * H * P * 2              # bf16
    dt = Bz * L * H * 4                     # f32
    bc = 2 * Bz * L * G * N * 2             # B and C, bf16
    ad = 2 * H * 4                          # A and D
    states = 2 * Bz * H * N * P * 4         # initial and final, f32
    want = x + y + dt + bc + ad + states
    assert bench.algorithmic_bytes(wl) == want
    assert abs(want / 1e9 - 2.835) < 0.01   # about 270 bytes per token-head
    assert abs(want / (Bz * L * H) - 270.4) < 0.5


def test_algorithmic_flops_of_the_2p7b_layer():
    wl = inputs.WORKLOADS["mamba2_2p7b_layer"]
    Bz, L, H, P, N, G, Q = 8, 16384, 80, 64, 128, 1, 256
    # causal MACs per token-head: C B^T (Q N / 2, shared by H / G heads), (S.L) X (Q P / 2),
    # chunk state (N P) and the inter-chunk product (N P)
    mac = Q * N / 2 / (H / G) + Q * P / 2 + N * P + N * P
    want = 2 * mac * Bz * L * H
    assert bench.algorithmic_flops(wl) == pytest.approx(want)
    assert want == pytest.approx(5.20e11, rel=0.01)


def test_l2_rule():
    # inputs under 256 MiB are flushed between steps; the headline's 2.8 GB are not
    assert bench.l2_resident(inputs.WORKLOADS["tiny_f32"])
    assert bench.l2_resident(inputs.WORKLOADS["mamba2_130m_layer"])
    assert not bench.l2_resident(inputs.WORKLOADS["mamba2_2p7b_layer"])
    assert not bench.l2_resident(inputs.WORKLOADS["long_context_layer"])
