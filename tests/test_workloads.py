"""Host-side workload plumbing (no GPU): the roofline-sweep workload names and
the bound on the oracle's timed sample in bench.py."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("shape", synth.SWEEP_SHAPES)
def test_sweep_workload_holds_one_gib_of_weights(shape):
    rows, cols = shape
    wl = synth.workload(f"sweep_{rows}x{cols}")
    assert all((m.rows, m.cols) == shape for m in wl.matrices)
    fp32_bytes = 4 * sum(m.size for m in wl.matrices)
    assert 1 << 30 <= fp32_bytes < (1 << 30) + 4 * rows * cols     # the smallest such batch
    assert wl.ns_steps == 5 and wl.ns_coeffs == (3.4445, -4.7750, 2.0315)
    assert set(wl.lrs) == {0.01}


@pytest.mark.parametrize("name", ["sweep_3x3", "sweep_512", "sweep_axb", "sweep_512x512x1"])
def test_unknown_sweep_names_are_refused(name):
    with pytest.raises(KeyError):
        synth.workload(name)


def test_cpu_sample_is_layer_zero_of_the_qwen3_sets():
    for name in ("qwen3_1.7b", "qwen3_0.6b"):
        wl, shapes = bench.workload_desc(name)
        assert bench.cpu_sample(shapes, wl.ns_steps) == list(range(7))
        assert {m.name.rsplit(".", 1)[0] for m in wl.matrices[:7]} == {"layers.0"}


@pytest.mark.parametrize("shape", synth.SWEEP_SHAPES)
def test_cpu_sample_stays_within_its_flop_bound(shape):
    wl, shapes = bench.workload_desc("sweep_%dx%d" % shape)
    idx = bench.cpu_sample(shapes, wl.ns_steps)
    assert idx == list(range(len(idx))) and 1 <= len(idx) <= 7
    flops = bench.ns_flops([shapes[i] for i in idx], wl.ns_steps)
    assert len(idx) == 1 or flops <= bench.CPU_SAMPLE_FLOPS
    if len(idx) < 7:       # one more matrix would break the bound
        assert bench.ns_flops(shapes[:len(idx) + 1], wl.ns_steps) > bench.CPU_SAMPLE_FLOPS
