"""The trace summaries of chunked_state_space_b200.pipeline_trace on synthetic
event clocks (CPU only): medians between events in the steady state and the
spread of CTA durations over the SMs."""
import numpy as np

from chunked_state_space_b200 import pipeline_trace, ssd


def test_summarize_reads_the_event_columns():
    E = {name: i for i, name in enumerate(ssd.TRACE_EVENTS)}
    n = 64
    t = np.zeros((n, 24), dtype=np.int64)
    base = np.arange(n) * 1000                       # a 1000-clock period
    t[:, E["loads"]] = base
    t[:, E["S_ready"]] = base + 300
    t[:, E["S_issued"]] = base + 350
    t[:, E["mask_start"]] = base + 400
    t[:, E["mask_done"]] = base + 650
    t[:, E["c_ready"]] = base + 700
    t[:, E["c_issued"]] = base + 800
    t[:, E["c_seen"]] = base + 900
    t[:, E["state_pub"]] = base + 950
    t[:, E["epi_done"]] = base + 990
    out = pipeline_trace.summarize(t)
    assert out["period (products issued, j -> j+1)"] == 1000
    assert out["loads issued -> S ready"] == 300
    assert out["mask start -> mask done"] == 250
    assert out["products ready -> issued"] == 100
    assert out["state published -> epilogue done"] == 40


def test_cta_summary_fill_of_the_sms():
    # 4 SMs, 6 CTAs of 100 us: two waves, the second half full
    ctas = np.array([[0, 100_000, 0], [0, 100_000, 1], [0, 100_000, 2], [0, 100_000, 3],
                     [100_000, 200_000, 0], [100_000, 200_000, 1]], dtype=np.int64)
    out = pipeline_trace.cta_summary(ctas)
    assert out["kernel span us"] == 200.0
    assert out["CTAs per SM (max)"] == 2
    assert out["SMs used"] == 4
    assert abs(out["sum of CTA time / (SMs x span)"] - 600.0 / 800.0) < 1e-12
