"""Host checks of bench.py's byte and flop models (no GPU).

The window model must reduce to the plain step's bytes for a window of one
step (a one-step window is the plain step), and must count exactly what the
window path moves: page, inputs and t rows each of K and D plus P read;
o, P', K[0..t], D[t] written, or codes and r at the commit.  The byte counts
of the packed page agree with the oracle's layout.
"""
import pytest

import bench
import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_window_of_one_is_the_plain_step(name):
    spec = W.FORMATS[name]
    assert bench.window_bytes_per_page(spec, 1) == bench.algorithmic_bytes_per_page(spec)


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_window_model_counts_each_position(name):
    spec = W.FORMATS[name]
    fmt = O.format_from_spec(spec)
    page = O.page_bytes(fmt)
    c = 512 if spec["col_scales"] else 0
    store = page - c                                   # codes + r
    inputs = 3 * 512 + (512 if spec["gate_vector"] else 4) + 4
    W_ = 4
    expect = 0
    for t in range(W_):
        read = page + inputs + (512 * (1 + 2 * t) if t > 0 else 0)
        write = 512 + (store if t == W_ - 1 else 512 * (t + 3))
        expect += read + write
    assert bench.window_bytes_per_page(spec, W_) == expect / W_
    # a window moves fewer bytes per step than the plain step while the buffer is short
    assert bench.window_bytes_per_page(spec, 4) < bench.algorithmic_bytes_per_page(spec)


def test_plain_step_bytes_match_the_page_layout():
    for name, spec in W.FORMATS.items():
        fmt = O.format_from_spec(spec)
        page = O.page_bytes(fmt)
        c = 512 if spec["col_scales"] else 0
        inputs = 3 * 512 + (512 if spec["gate_vector"] else 4) + 4 + 512
        assert bench.algorithmic_bytes_per_page(spec) == 2 * (page - c) + c + inputs, name


def test_prefill_flops_and_peak():
    assert bench.prefill_flops_per_head_token() == 128 * 128 * 7
    assert abs(bench.FP32_PEAK_TFLOPS - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9


@pytest.mark.parametrize("k", [1, 2, 3, 5, 7, 20, 2000, 2003])
def test_repetitions_cover_exactly_the_timed_steps(k):
    sizes = bench.split_reps(k)
    assert sum(sizes) == k
    assert len(sizes) == min(5, k)
    assert max(sizes) - min(sizes) <= 1


def test_roofline_object_against_both_peaks():
    spec = W.FORMATS["damp"]
    pages, ms = 131072, 1.5
    r = bench.hbm_roofline(spec, pages, ms, "damp-gdn")
    gbs = bench.algorithmic_bytes_per_page(spec) * pages / (ms / 1000.0) / 1e9
    assert abs(r["achieved"] - gbs) < 1e-9 * gbs
    assert abs(r["frac"] - gbs / r["peak"]) < 1e-12
    assert abs(r["frac_of_nominal_8tbs"] - gbs / 8000.0) < 1e-12
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
