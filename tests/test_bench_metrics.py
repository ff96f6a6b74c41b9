"""The numbers bench.py derives around its timings, checked on the CPU.

Every fraction the benchmark reports divides a measured time into counts
that do not depend on the GPU: the live pairs of the pattern (nnz), the
useful flops (14 d nnz, 12 d nnz without the recomputed S), the fewest HBM
bytes a kernel or a step can move, and the roofline those give. These tests
check them against the closed-form pair totals in tests/golden/nnz.json and
against the byte counts written out by hand."""
import json
import os

import pytest

import bench
import factorized_sparse_self_b200 as st
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nnz.json")


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_nnz_matches_the_closed_form_totals(name):
    w = synth.WORKLOADS[name]
    gold = json.load(open(GOLDEN))["workloads"][name]
    L = st.st_pattern_layout_host(w.kind, w.mode, w.T, w.l, w.c)
    assert bench.nnz_of(L, w) == gold["total"]


def test_headline_byte_counts():
    w = synth.WORKLOADS["fixed-split-T4096"]
    rows = 4 * 8 * 4096
    row = 64 * 2  # one bf16 row of d = 64
    # forward: Q, K, V read, O written (bf16), LSE written (fp32)
    assert bench.fwd_bytes(w) == rows * row * 4 + rows * 4
    # backward kernel: Q, K, V, dO read, dQ, dK, dV written, LSE and D read
    assert bench.bwd_bytes(w) == rows * row * 7 + rows * 4 * 2 == 118489088
    # whole step: the forward's bytes plus Q, K, V, O, dO, LSE read and
    # dQ, dK, dV written by the backward
    assert bench.step_min_bytes(w) == rows * row * 12 + rows * 4 * 2 == 202375168


def test_step_roofline_takes_the_lower_ceiling():
    w = synth.WORKLOADS["fixed-split-T4096"]
    flops = 14.0 * 64 * 18681856
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 1000.0}
    r = bench.step_roofline(w, flops, 1.0, peaks)
    intensity = flops / 202375168
    assert r["flop_per_byte"] == pytest.approx(intensity)
    assert r["bound"] == "hbm"
    assert r["roofline_tflops"] == pytest.approx(intensity * 1000e9 / 1e12)
    assert r["useful_tflops"] == pytest.approx(flops / 1e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["useful_tflops"] / r["roofline_tflops"])
    # with a slow tensor unit the same step is bound by it instead
    r2 = bench.step_roofline(w, flops, 1.0, {"bf16_tflops": 10.0, "hbm_gbs": 1000.0})
    assert r2["bound"] == "tensor" and r2["roofline_tflops"] == 10.0


def test_flop_counts_per_step():
    # 4 d nnz forward, 10 d nnz backward with the recomputed S (12 d nnz without)
    w = synth.WORKLOADS["fixed-split-T4096"]
    nnz = 18681856
    assert bench.whole_job_tflops(1, 14.0 * w.d * nnz, 1.0) == pytest.approx(16.738942976)
    assert bench.whole_job_tflops(1, 12.0 * w.d * nnz, 1.0) == pytest.approx(14.347665408)
