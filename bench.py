"""Throughput of the MoE layer hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gpt2] [--impl native|reference]

A step is one pass of the whole layer (route, scan, permute, expert up- and
down-projections, combine, statistics) over one batch of synthetic tokens
already resident in device memory.  One layer call (moe_forward_timed, which
records CUDA events between its stages on the launching stream) is captured
as a CUDA graph and replayed once per step, with events only around the
dominant stage (its duration gives the roofline figure); each step's time is
the span of two events recorded on the stream around the replay.  A separate
pass of up to 20 steps with an event between every two stages gives the stage
breakdown.  The L2 cache is flushed (a 512 MiB buffer is written) before
every step, outside the events.  `e2e` repeats the measurement through plain
moe_forward calls with the input copied in from pinned host memory and the
output and losses copied back, every step.  With N > 1 (torchrun) every rank runs
its own batch on its own GPU (weak scaling, no collective on the data path);
the reported time is the maximum over ranks.

`--impl reference` times the fp64 oracle on the host cores instead (the
reference arm of this comparison), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import ACT_GELU, ACT_SWIGLU, WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and active TFLOP/s (or GB/s at decode) vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_KERNEL_SRC = os.path.join(ROOT, "sparse_mixture_experts_10_b200", "csrc", "moe_gemm_tc.cuh")

# DRAM traffic of the dominant kernel per launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum); keyed by workload and stage,
# valid only while the kernel source hash is unchanged (see profiles/).
NCU_TRAFFIC = {
    "gpt2/up": {"bytes": 108708096, "src_sha256": "7c227d73ad4b51f9796bb92c7559833d64a345edf15e8706150dde12569545b6"},
    "gpt2/down": {"bytes": 184628992, "src_sha256": "7c227d73ad4b51f9796bb92c7559833d64a345edf15e8706150dde12569545b6"},
}


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: the per-GPU work is fixed)."""
    return wl.seed + 7919 * rank


def max_over_ranks(value_ms: float, device, world: int) -> float:
    """The job's time is the slowest rank's (all ranks take the same collective steps)."""
    if world == 1:
        return value_ms
    import torch.distributed as dist

    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: the tokens every rank processed over the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_total_ms / 1e3)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="gpt2", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def sha256(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def work_model(wl, T, counts=None):
    """Algorithmic work per layer call (routed rows only, no padding)."""
    D, H, N, K = wl.D, wl.H, wl.N, wl.K
    b = 4 if wl.dtype == torch.float32 else 2
    c_up = 4 if wl.act == ACT_SWIGLU else 2
    up_flops = T * K * c_up * D * H
    down_flops = T * K * 2 * D * H
    router_flops = T * 2 * D * N
    live = int((counts > 0).sum()) if counts is not None else min(N, T * K)
    up_rows = 2 * H if wl.act == ACT_SWIGLU else H
    # bf16 prefill with K <= 2 (y is fp32 here): the permute kernel clears y and
    # the down projection adds into it, so there is no combine pass
    fused_combine = b == 2 and T > 64 and K <= 2
    return dict(
        flops=router_flops + up_flops + down_flops,
        up_flops=up_flops, down_flops=down_flops, router_flops=router_flops,
        route_bytes=T * D * b + D * N * b + T * N * 4 + T * K * 8,
        permute_bytes=T * D * b + T * K * D * b + T * K * 8 + (T * D * 4 if fused_combine else 0),
        combine_bytes=0 if fused_combine else T * K * D * 4 + T * D * 4,
        up_weight_bytes=live * up_rows * D * b, down_weight_bytes=live * D * H * b,
        live_experts=live,
    )


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        self.p.wait(timeout=10)
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for k, name in enumerate(names):
                    if r[5 + k].strip().lower() == "active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_rate(wl, inp, budget_s):
    """The fp64 oracle, as it stands, on a bounded token sample on the host cores: tokens/s."""
    import oracle
    from moe_inputs import bf16_bits

    T = inp["x"].shape[0]
    threads = oracle.default_threads()
    tag = oracle.F32 if wl.dtype == torch.float32 else oracle.BF16
    h = {k: (None if v is None else bf16_bits(v)) for k, v in inp.items()}

    def run(a, b):
        oracle.moe_layer(h["x"][a:b], h["W_g"], h["W1"], h["W2"], K=wl.K, act=wl.act, dtype_tag=tag, bg=h["b_g"],
                         b1=h["b1"], b2=h["b2"], threads=threads)

    n = min(T, max(threads, 4))
    t0 = time.perf_counter()
    run(0, n)
    dt = time.perf_counter() - t0
    total_n, total_t = n, dt
    n2 = int(min(T - n, max(0, (budget_s - dt) / max(dt / n, 1e-9))))
    if n2 > 0:
        t0 = time.perf_counter()
        run(n, n + n2)
        total_t += time.perf_counter() - t0
        total_n += n2
    return total_n / total_t, threads, f"{total_n} of {T} tokens, whole layer (router, experts, combine), fp64"


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    torch.manual_seed(0)
    inp = make_inputs(wl, "cpu", seed=wl.seed)
    per_step = max(0.2, 60.0 / max(args.steps + args.warmup, 1))
    rates = []
    cores = 1
    sample = ""
    for i in range(args.warmup + args.steps):
        r, cores, sample = cpu_oracle_rate(wl, inp, per_step)
        if i >= args.warmup:
            rates.append(r)
    v = statistics.median(rates)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * wl.T / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "D": wl.D, "H": wl.H, "N": wl.N, "K": wl.K},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import torch.distributed as dist

    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    import sparse_mixture_experts_10_b200 as moe
    from sparse_mixture_experts_10_b200 import build as moe_build

    if rank == 0:
        moe_build.build()
    if world > 1:
        dist.barrier()
    moe.load_library()

    T = wl.T
    inp = make_inputs(wl, dev, seed=rank_seed(wl, rank))
    cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias)
    W = moe.make_weights(inp["W_g"], inp["W1"], inp["W2"], inp["b_g"], inp["b1"], inp["b2"])
    ws = moe.alloc_workspace(cfg, T)
    y = torch.empty(T, wl.D, dtype=torch.float32, device=dev)
    aux_t = dict(counts=torch.empty(wl.N, dtype=torch.int32, device=dev),
                 importance=torch.empty(wl.N, device=dev), p_mean=torch.empty(wl.N, device=dev),
                 scalars=torch.empty(4, device=dev))
    aux = moe.make_aux(**aux_t)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    NS = moe.MOE_N_STAGES

    def step(evs, strm=None):
        moe.check(moe.moe_forward_timed(cfg, inp["x"], T, W, y, moe.MOE_F32, aux, ws, ws.numel(),
                                        strm or torch.cuda.current_stream(dev), evs), "forward")

    warm = [torch.cuda.Event(enable_timing=True) for _ in range(NS + 1)]
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step(warm)
    torch.cuda.synchronize()
    st = moe.moe_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    counts = aux_t["counts"].cpu().numpy()

    def capture(stage_events):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(stage_events)
        return g

    def new_events(n):
        out = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in out:
            e.record()
        return out

    # Stage breakdown: one layer call with an event between every two stages,
    # captured as a CUDA graph and replayed (each event node adds a few
    # microseconds, so these steps are not the timed ones).
    evs = new_events(NS + 1)
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    graph = capture(evs)
    launches_per_step = moe.moe_launch_count() - l0
    rows = []
    n_break = min(args.steps, 20)
    for i in range(2 + n_break):
        flush.zero_()
        graph.replay()
        torch.cuda.synchronize()
        if i >= 2:
            rows.append([evs[s_].elapsed_time(evs[s_ + 1]) for s_ in range(NS)])
    del graph
    stage_ms = np.array(rows)
    mean_stage = stage_ms.mean(axis=0)
    names = moe.STAGE_NAMES
    dom = int(np.argmax(mean_stage))

    # Timed steps: the layer call as a graph with events only around the
    # dominant stage (its duration for the roofline); the step time is taken
    # by events recorded on the stream around each replay.
    dom_ev = [None] * (NS + 1)
    dom_ev[dom], dom_ev[dom + 1] = new_events(2)
    step_ev = [tuple(new_events(2)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    graph = capture(dom_ev)
    for _ in range(2):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, dom_ms = [], []
    for i in range(args.steps):
        flush.zero_()
        step_ev[i][0].record(stream)
        graph.replay()
        step_ev[i][1].record(stream)
        torch.cuda.synchronize()
        step_ms.append(step_ev[i][0].elapsed_time(step_ev[i][1]))
        dom_ms.append(dom_ev[dom].elapsed_time(dom_ev[dom + 1]))
    launches = launches_per_step * args.steps
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st = moe.moe_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")
    del graph

    total_ms = max_over_ranks(float(sum(step_ms)), dev, world)
    ms_per_step = total_ms / args.steps
    tokens_per_s = job_throughput(T, world, args.steps, total_ms)
    dom_mean_ms = float(np.mean(dom_ms))

    # ---- end to end through host buffers: pinned x in, y and the statistics out, every step
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty(T, wl.D, dtype=torch.float32).pin_memory()
    sc_host = torch.empty(4).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(max(args.warmup, 3) + args.steps):
        flush.zero_()
        if i >= max(args.warmup, 3):
            e2e_ev[i - max(args.warmup, 3)][0].record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        moe.check(moe.moe_forward(cfg, x_dev, T, W, y, moe.MOE_F32, aux, ws, ws.numel(), stream))
        y_host.copy_(y, non_blocking=True)
        sc_host.copy_(aux_t["scalars"], non_blocking=True)
        if i >= max(args.warmup, 3):
            e2e_ev[i - max(args.warmup, 3)][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), dev, world)
    e2e_tps = job_throughput(T, world, args.steps, e2e_ms)
    es = x_host.element_size()
    h2d = T * wl.D * es
    d2h = T * wl.D * 4 + 16

    # ---- roofline of the dominant kernel (its duration from the timed steps)
    wm = work_model(wl, T, counts)
    pk, pk_kind = peaks()
    decode = wl.name.startswith("decode")
    if names[dom] in ("up", "down") and not decode:
        fl = wm["up_flops"] if names[dom] == "up" else wm["down_flops"]
        achieved = fl / (dom_mean_ms * 1e-3) / 1e12
        peak = float(pk["bf16_tflops"])
        roof = {"kernel": f"grouped_gemm_tc ({names[dom]})", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": f"{pk_kind} bf16 burst"}
    else:
        byt = {"route": wm["route_bytes"], "permute": wm["permute_bytes"], "combine": wm["combine_bytes"],
               "up": wm["up_weight_bytes"], "down": wm["down_weight_bytes"]}.get(names[dom], 0)
        achieved = byt / (dom_mean_ms * 1e-3) / 1e9
        peak = float(pk["hbm_gbs"])
        roof = {"kernel": names[dom], "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"{pk_kind} copy"}
    roof["ms"] = dom_mean_ms
    key = f"{wl.name}/{names[dom]}"
    tr = NCU_TRAFFIC.get(key)
    roof["traffic"] = tr["bytes"] if tr and tr["src_sha256"] == sha256(GEMM_KERNEL_SRC) else None

    stages = {}
    for s, nm in enumerate(names):
        d = {"ms": float(mean_stage[s])}
        if nm == "route":
            d["GB/s"] = wm["route_bytes"] / (mean_stage[s] * 1e-3) / 1e9
        elif nm == "permute":
            d["GB/s"] = wm["permute_bytes"] / (mean_stage[s] * 1e-3) / 1e9
        elif nm == "combine":
            d["GB/s"] = wm["combine_bytes"] / (mean_stage[s] * 1e-3) / 1e9
        elif nm in ("up", "down"):
            fl = wm["up_flops"] if nm == "up" else wm["down_flops"]
            d["TFLOP/s"] = fl / (mean_stage[s] * 1e-3) / 1e12
            d["weight GB/s"] = (wm["up_weight_bytes"] if nm == "up" else wm["down_weight_bytes"]) / (
                mean_stage[s] * 1e-3) / 1e9
        stages[nm] = d

    line = {"metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": {"workload": wl.name, "T": T, "D": wl.D, "H": wl.H, "N": wl.N, "K": wl.K,
                       "act": "swiglu" if wl.act == ACT_SWIGLU else "gelu", "global_batch": T * world,
                       "parallelism": f"dp{world}", "l2": "flushed (512 MiB write) before every step"},
            "active_tflops": wm["flops"] * world * args.steps / (total_ms / 1e3) / 1e12,
            "roofline": roof, "stages": stages,
            "stages_note": f"{n_break} separate steps with an event between every two stages",
            "e2e": {"value": e2e_tps, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_rate(wl, inp, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
