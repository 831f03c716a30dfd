"""Host-side pieces of bench.py that need no GPU: the reference arm's steps
are an exact partition of a layer call, the whole-job throughput, the
encoder workloads' block formats and the algorithmic byte counts."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("q4k", [False, True])
def test_reference_steps_partition_one_layer_call(q4k):
    """F steps of the reference arm's sampler, one per row block, sum to the
    oracle's whole layer output for the same tokens."""
    s = synth.LayerShape(256, 256, 256, 32, 2, 1, vocab=1024, q4k=q4k)
    smp = bench.OracleSampler(s)
    for _ in range(smp.F):
        smp.step()
    W = smp.W
    ref = oracle.layer(W, s, smp.x, smp.idx, smp.w)
    assert np.allclose(smp.y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())
    assert smp.tokens_per_step * smp.F == smp.T


def test_job_throughput_and_formats():
    assert bench.job_throughput(4, 10, 8, 20.0) == pytest.approx(4 * 10 * 8 / 0.020)
    assert bench.quant_format("quantize_q2k") == (1, 256, 84)
    assert bench.quant_format("quantize_q4k") == (2, 256, 144)
    assert bench.quant_format("quantize_q80") == (0, 32, 34)


def test_decode_bytes_follow_the_routed_format():
    s = synth.workload("decode_t1")
    b = bench.decode_bytes(s, 6.0)
    assert b["k2_experts"] == 69_206_016  # six q2 experts and the shared expert (page figures)
    s4 = synth.workload("decode_t1_q4k")
    assert bench.decode_bytes(s4, 6.0)["experts"] == 6 * 3 * 4096 * 2048 * 144 // 256 + 26_738_688


def test_box_fractions():
    """The box-measured and nominal fractions divide the roofline's achieved
    figure by the peak of its own unit, and leave the pool's frac alone."""
    line = {"roofline": {"achieved": 1600.0, "unit": "GB/s", "frac": 0.24}}
    bench.add_box_fracs(line, {"copy_gbs": 6400.0, "bf16_tflops": 1500.0})
    r = line["roofline"]
    assert r["frac_of_box_peak"] == pytest.approx(0.25)
    assert r["frac_of_nominal"] == pytest.approx(0.2)
    assert r["frac"] == 0.24
    line = {"roofline": {"achieved": 450.0, "unit": "TFLOP/s"}}
    bench.add_box_fracs(line, {"error": "no GPU"})
    assert "frac_of_box_peak" not in line["roofline"]
    assert line["roofline"]["frac_of_nominal"] == pytest.approx(0.2)
