"""Host-side arithmetic of bench.py: the algorithmic work per layer call that every
roofline figure divides by, and the peaks it divides into."""
import os

import numpy as np
import pytest

import bench
from moe_inputs import WORKLOADS


def test_gpt2_work_model_counts():
    wl = WORKLOADS["gpt2"]
    T, D, H, N, K = wl.T, wl.D, wl.H, wl.N, wl.K
    m = bench.work_model(wl, T)
    # GELU expert: two GEMMs of 2*D*H FLOPs per routed row; router 2*D*N per token
    assert m["up_flops"] == 2 * T * K * D * H
    assert m["down_flops"] == 2 * T * K * D * H
    assert m["flops"] == 2 * T * D * N + 4 * T * K * D * H
    # bf16 prefill with K = 2 and an fp32 y: the permute pass also clears y, and there is no combine pass
    assert m["permute_bytes"] == T * D * 2 + T * K * D * 2 + T * K * 8 + T * D * 4
    assert m["combine_bytes"] == 0
    assert m["live_experts"] == N
    assert m["up_weight_bytes"] == N * H * D * 2


def test_swiglu_and_separate_combine_work_model():
    wl = WORKLOADS["deepseek"]   # K = 8: the combine is a pass of its own
    T, D, H, N, K = wl.T, wl.D, wl.H, wl.N, wl.K
    m = bench.work_model(wl, T)
    assert m["up_flops"] == 4 * T * K * D * H          # gate and up
    assert m["down_flops"] == 2 * T * K * D * H
    assert m["combine_bytes"] == T * K * D * 4 + T * D * 4
    assert m["permute_bytes"] == T * D * 2 + T * K * D * 2 + T * K * 8


def test_decode_reads_only_live_experts():
    wl = WORKLOADS["decode1"]
    counts = np.zeros(wl.N, dtype=np.int64)
    counts[[3, 7, 11, 30]] = 1
    m = bench.work_model(wl, wl.T, counts)
    assert m["live_experts"] == 4
    assert m["up_weight_bytes"] == 4 * 2 * wl.H * wl.D * 2      # packed gate_up rows, bf16
    assert m["down_weight_bytes"] == 4 * wl.D * wl.H * 2
    assert m["combine_bytes"] == wl.T * wl.K * wl.D * 4 + wl.T * wl.D * 4   # decode keeps its combine pass


def test_peaks_come_from_the_measured_file_when_present():
    pk, kind = bench.peaks()
    path = os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "MEASURED_PEAKS.json")
    if os.path.exists(path):
        assert kind == "measured"
        assert pk["hbm_gbs"] > 0 and pk["bf16_tflops"] > 0
    else:
        assert kind == "fallback"
        assert pk["hbm_gbs"] == pytest.approx(6650.0) and pk["bf16_tflops"] == pytest.approx(1590.0)
