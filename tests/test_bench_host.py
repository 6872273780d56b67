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
    # bf16 prefill with K = 2 and an fp32 y: the SIMT router (N <= 32) clears y, the down
    # projection adds into it, and there is no combine pass
    assert bench.simt_router_clears_y(wl, T)
    assert m["route_bytes"] == T * D * 2 + D * N * 2 + T * N * 4 + T * K * 8 + T * D * 4
    assert m["permute_bytes"] == T * D * 2 + T * K * D * 2 + T * K * 8
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


def test_permute_clears_y_when_the_router_is_not_the_simt_one():
    from moe_inputs import Workload, ACT_SWIGLU
    import torch
    wl = Workload("many", 11, 700, 256, 128, 64, 2, ACT_SWIGLU, torch.bfloat16, False, 0.05)
    m = bench.work_model(wl, wl.T)
    T, D, K, N = wl.T, wl.D, wl.K, wl.N
    assert not bench.simt_router_clears_y(wl, T)
    assert m["permute_bytes"] == T * D * 2 + T * K * D * 2 + T * K * 8 + T * D * 4
    assert m["route_bytes"] == T * D * 2 + D * N * 2 + T * N * 4 + T * K * 8


def test_default_workload_is_the_largest_single_gpu_config():
    args = bench.parse([])
    assert args.workload == "deepseek" and args.gpus == 1
    assert args.warmup >= 3
    wl = WORKLOADS[args.workload]
    assert bench.expert_weight_bytes(wl) == max(bench.expert_weight_bytes(w) for w in WORKLOADS.values())


def test_gemm_peak_is_sustained_inside_long_steps():
    pk = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    assert bench.gemm_peak(pk, 14.0) == (1400.0, "bf16 sustained")
    assert bench.gemm_peak(pk, 0.19) == (1650.0, "bf16 burst")


def test_decode_bytes_cover_live_experts_and_activations():
    wl = WORKLOADS["decode8"]
    counts = np.zeros(wl.N, dtype=np.int64)
    counts[:21] = 1
    m = bench.work_model(wl, wl.T, counts)
    D, H, N, T = wl.D, wl.H, wl.N, wl.T
    assert m["decode_bytes"] == 21 * (2 * H * D + D * H) * 2 + T * D * 2 + T * D * 4 + D * N * 2


@pytest.mark.parametrize("whole", [True, False])
def test_oracle_sample_rates_and_labels(whole, monkeypatch):
    """The CPU baseline runs the oracle as it stands on a bounded sample: whole tokens, or (for
    layers with many GB of experts) the router on sampled tokens and the experts on sampled
    (token, slot) pairs of a few experts."""
    from moe_inputs import make_inputs
    if not whole:
        monkeypatch.setattr(bench, "WHOLE_LAYER_WEIGHT_BYTES", 0)
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cpu", T=128)
    smp = bench.OracleSample(wl, inp, seed=3, threads=2)
    assert smp.whole == whole
    r0, wall0, cores0, desc0 = smp.step(0.05)
    r1, wall1, cores1, desc1 = smp.step(0.2)
    assert r0 > 0 and r1 > 0 and wall1 > 0 and 1 <= cores1 <= 2
    assert ("(token, slot) pairs" in desc1) != whole
    if not whole:
        assert "pairs" in desc1 and "extrapolated" in desc1
        assert len(smp.ew) <= 8 and all(e in smp.ew for _, e in smp.pairs)


def test_reference_arm_line(capsys):
    """--impl reference: the oracle's line carries the native arm's config, an honest step time
    (what the step ran) and the extrapolated whole-layer time apart."""
    import json
    args = bench.parse(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "1",
                        "--ref-seconds", "2"])
    bench.run_reference(args, WORKLOADS["tiny"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["extrapolated"] is True
    assert line["config"] == bench.config_dict(WORKLOADS["tiny"], WORKLOADS["tiny"].T, 1)
    assert line["ms_per_step"] > 0 and line["ms_per_layer_extrapolated"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reduced_profiling_case_keeps_the_shape_per_expert():
    args = bench.parse(["--workload", "deepseek", "--tokens", "2048", "--experts", "32"])
    wl = bench.workload_from_args(args)
    full = WORKLOADS["deepseek"]
    assert (wl.T, wl.N, wl.D, wl.H, wl.K) == (2048, 32, full.D, full.H, full.K)
    assert wl.T * wl.K // wl.N == full.T * full.K // full.N      # 512 assignments per expert either way
    assert wl.name.startswith("deepseek[")
    assert bench.workload_from_args(bench.parse([])) == WORKLOADS["deepseek"]


def test_capacity_counts_only_the_kept_pairs():
    """With a per-expert capacity the dropped (token, slot) pairs cost no expert work: FLOPs,
    copies and combine reads follow the accepted pairs, the slot maps all T*K pairs."""
    wl = WORKLOADS["deepseek_zipf"].with_(capacity_factor=1.0)
    T, D, H, N, K = wl.T, wl.D, wl.H, wl.N, wl.K
    kept = np.zeros(N, dtype=np.int64)
    kept[:40] = 512                       # 40 experts full at C = T*K/N, the rest dropped
    rows = 40 * 512
    m = bench.work_model(wl, T, np.full(N, T * K // N), kept)
    assert m["up_flops"] == 4 * rows * D * H
    assert m["down_flops"] == 2 * rows * D * H
    assert m["flops"] == 2 * T * D * N + 6 * rows * D * H
    assert m["permute_bytes"] == T * D * 2 + rows * D * 2 + T * K * 8
    assert m["combine_bytes"] == rows * D * 4 + T * D * 4
    assert m["live_experts"] == 40
    # without a capacity every routed pair is work
    assert bench.work_model(wl, T)["up_flops"] == 4 * T * K * D * H


def test_permute_write_bytes_are_the_copies_and_any_clear_of_y():
    wl = WORKLOADS["deepseek"]   # K = 8: the permute writes the copies, nobody clears y
    T, D, K = wl.T, wl.D, wl.K
    m = bench.work_model(wl, T)
    assert m["permute_write_bytes"] == T * K * D * 2
    assert m["permute_bytes"] - m["permute_write_bytes"] == T * D * 2 + T * K * 8
    wl = WORKLOADS["mixtral"]    # K = 2, N <= 32: the SIMT router clears y, not the permute
    m = bench.work_model(wl, wl.T)
    assert m["permute_write_bytes"] == wl.T * wl.K * wl.D * 2
