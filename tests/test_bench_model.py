"""The bench's work model: layer FLOPs against their closed form and the per-workload totals
(K counts partial edge cubes), and the cube counts the bench divides by."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("name,K,flops", [("tiny", 64, 4.61e7), ("wan480p_proj", 8190, 2.168e12),
                                          ("wan720p_ffn_up", 10120, 1.223e13),
                                          ("wan720p_ffn_down", 19320, 1.353e13)])
def test_layer_flops(name, K, flops):
    wl = synth.WORKLOADS[name]
    assert oracle.num_cubes(wl.T, wl.H, wl.W, *wl.cube) == K
    F = bench.layer_flops(wl, K)
    N, Ci, Co, r = wl.N, wl.Ci, wl.Co, wl.rank
    assert F == 2.0 * N * Ci * Co + 2.0 * K * Ci * Co + 2.0 * N * r * (Ci + Co)
    assert F == pytest.approx(flops, rel=2e-3)


def test_stage_model_counts_both_reads_of_x():
    wl = synth.WORKLOADS["wan480p_proj"]
    m = bench.stage_model(wl, 8190, 64)
    assert m["quantize"]["bytes"] >= 4.0 * wl.N * wl.Ci          # X read by both passes
    assert m["main_gemm"]["flops"] == 2.0 * wl.N * wl.Ci * wl.Co + 2.0 * wl.N * 64 * wl.Co
    assert m["kernel_gemm"]["flops"] == 2.0 * 8190 * wl.Ci * wl.Co
    g = bench.stage_model(wl, 8190, 64, kernel_group=64)
    assert g["kernel_gemm"]["bytes"] > m["kernel_gemm"]["bytes"]  # hi + lo operand


def test_cpu_baseline_sample():
    """The CPU baseline's cube sample: the whole tensor for the small layers, else
    512 distinct seeded cubes, the same on every call; per-row FLOPs add up to the
    layer's."""
    wl = synth.WORKLOADS["wan720p_ffn_down"]
    a, full = bench.oracle_sample_cubes(wl, wl.cube)
    b, _ = bench.oracle_sample_cubes(wl, wl.cube)
    assert not full and a.size == 512 == np.unique(a).size and np.array_equal(a, b)
    assert a.min() >= 0 and a.max() < 19320
    t, full_t = bench.oracle_sample_cubes(synth.WORKLOADS["tiny"], (1, 2, 2))
    assert full_t and np.array_equal(t, np.arange(64))
    assert bench.layer_flops_rows(wl, 19320, wl.N) == pytest.approx(bench.layer_flops(wl, 19320), rel=1e-12)
