"""Throughput of the MoE layer hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload deepseek] [--impl native|reference]

A step is one pass of the whole layer (route, scan, permute, expert up- and
down-projections, combine, statistics) over one batch of synthetic tokens
already resident in device memory.  The default workload is the largest
single-GPU one, the DeepSeek-V3-shaped layer (T=16384, D=7168, H=2048, 256
experts, top-8, SwiGLU); ``--workload`` selects the others.

One layer call (moe_forward_timed, which records CUDA events between its
stages on the launching stream) is captured as a CUDA graph and replayed once
per step, with events only around the dominant stage (its duration gives the
roofline figure); each step's time is the span of two events recorded on the
stream around the replay.  A separate pass of up to 20 steps with an event
between every two stages gives the stage breakdown.  The L2 cache is flushed
(a 512 MiB buffer is written) before every step, outside the events.

``e2e`` is the same metric through plain moe_forward calls with host buffers:
each step copies its input in from pinned host memory and copies y and the
loss scalars back, on copy streams of their own, so that the copies of one
step overlap the kernels of its neighbours (double-buffered x, y and
statistics).  Its time runs from the first copy-in to the last copy-out.

With N > 1 (torchrun) every rank runs its own batch on its own GPU (weak
scaling) and the layer's statistics are made global: each rank's exact
integer partial sums are all-reduced (NCCL) and finalised identically on every
rank.  The reported time is the maximum over ranks.

``--impl reference`` times the fp64 oracle on the host cores instead (the
reference arm of this comparison), on a bounded sample of the same workload;
the result is extrapolated to the whole batch (tokens are independent) and
labelled so.
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
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import ACT_GELU, ACT_SWIGLU, WORKLOADS, bf16_bits, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and active TFLOP/s (or GB/s at decode) vs B200 roofline"
DEFAULT_WORKLOAD = "deepseek"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures: dense bf16 tensor throughput and HBM3e bandwidth
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
# steps longer than this run the tensor cores long enough to sit under the power cap:
# the GEMM roofline then uses the measured sustained figure instead of the burst one
SUSTAINED_STEP_MS = 1.0
# above this many bytes of expert weights the oracle sample evaluates (token, slot)
# pairs of a few experts instead of whole tokens (only those experts go to the host)
WHOLE_LAYER_WEIGHT_BYTES = 4 << 30
GEMM_KERNEL_SRC = os.path.join(ROOT, "sparse_mixture_experts_10_b200", "csrc", "moe_gemm_tc.cuh")

# DRAM bytes per launch of the dominant pair GEMM (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the source with this hash: the GPT-2-width layer captured as is; the DeepSeek-V3
# layer from the reduced case of 2048 tokens and 32 experts (512 rows per expert as at full size),
# scaled by 8 (weights and token rows both grow eightfold).  The tail kernel beside the pair kernel
# is not included.  Keyed by workload and stage; valid only while the source hash is unchanged.
NCU_TRAFFIC = {
    "gpt2/up": {"bytes": 54389760 + 53961216, "src_sha256": "410a9cd9ccbbf5b3802a66ad2371756e66bd410e05e0ccfb4cedcff2781a330b"},
    "gpt2/down": {"bytes": 166587136 + 10543360, "src_sha256": "410a9cd9ccbbf5b3802a66ad2371756e66bd410e05e0ccfb4cedcff2781a330b"},
    "deepseek/up": {"bytes": 8 * (2115678000 + 66724608), "src_sha256": "410a9cd9ccbbf5b3802a66ad2371756e66bd410e05e0ccfb4cedcff2781a330b",
                    "note": "scaled from the T=2048, N=32 capture"},
    "deepseek/down": {"bytes": 8 * (1008105000 + 440681728), "src_sha256": "410a9cd9ccbbf5b3802a66ad2371756e66bd410e05e0ccfb4cedcff2781a330b",
                      "note": "scaled from the T=2048, N=32 capture"},
}


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own tokens (weak scaling: the per-GPU work is fixed)."""
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


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--mode", default="forward", choices=["forward", "backward", "route"],
                    help="backward: time the layer's backward pass (moe_backward) instead; route: the "
                         "routing stage alone (moe_route)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="target CPU time of the whole --impl reference run (all steps)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="reduced case for profiling: override the workload's token count")
    ap.add_argument("--experts", type=int, default=0,
                    help="reduced case for profiling: override the number of experts (tokens per expert kept "
                         "when --tokens is scaled with it)")
    ap.add_argument("--capacity-factor", type=float, default=None,
                    help="per-expert capacity ceil(cf T K / N) (default: the workload's own)")
    ap.add_argument("--overflow", default=None, choices=["drop", "reroute"],
                    help="what a full expert does with a further assignment (with a capacity)")
    return ap.parse_args(argv)


def workload_from_args(args):
    """The named workload, or its reduced profiling case (--tokens / --experts)."""
    wl = WORKLOADS[args.workload]
    kw = {}
    if args.tokens:
        kw["T"] = args.tokens
    if args.experts:
        kw["N"] = args.experts
    if getattr(args, "capacity_factor", None) is not None:
        kw["capacity_factor"] = args.capacity_factor
    if getattr(args, "overflow", None) is not None:
        kw["overflow"] = 1 if args.overflow == "reroute" else 0
    if kw:
        wl = wl.with_(name=f"{wl.name}[" + ",".join(f"{k}={v}" for k, v in kw.items()) + "]", **kw)
    return wl


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


def expert_weight_bytes(wl) -> int:
    b = 4 if wl.dtype == torch.float32 else 2
    rows1 = 2 * wl.H if wl.act == ACT_SWIGLU else wl.H
    return wl.N * (rows1 * wl.D + wl.D * wl.H) * b


def fused_combine(wl, T) -> bool:
    """bf16 prefill with K <= 2 and an fp32 y: the down projection adds into y, no combine pass."""
    return wl.dtype == torch.bfloat16 and T > 64 and wl.K <= 2


def simt_router_clears_y(wl, T) -> bool:
    """Which kernel clears y for the folded combine: the SIMT router (bf16, N <= 32, T > 64),
    else the permute kernel."""
    return fused_combine(wl, T) and wl.N <= 32


def work_model(wl, T, counts=None, kept=None):
    """Algorithmic work per layer call (routed rows only, no padding), per stage.  With a
    per-expert capacity, kept holds each expert's accepted (token, slot) pairs: only those rows
    are copied, multiplied and combined (a dropped pair costs no expert work)."""
    D, H, N, K = wl.D, wl.H, wl.N, wl.K
    b = 4 if wl.dtype == torch.float32 else 2
    c_up = 4 if wl.act == ACT_SWIGLU else 2
    rows = int(np.asarray(kept).sum()) if kept is not None else T * K
    if kept is not None:
        live = int((np.asarray(kept) > 0).sum())
    else:
        live = int((np.asarray(counts) > 0).sum()) if counts is not None else min(N, T * K)
    up_flops = rows * c_up * D * H
    down_flops = rows * 2 * D * H
    router_flops = T * 2 * D * N
    up_rows = 2 * H if wl.act == ACT_SWIGLU else H
    y_clear = T * D * 4 if fused_combine(wl, T) else 0
    by_router = simt_router_clears_y(wl, T)
    return dict(
        flops=router_flops + up_flops + down_flops,
        up_flops=up_flops, down_flops=down_flops, router_flops=router_flops,
        # x, W_g, logits, top-k indices and weights (+ the clear of y when the router does it)
        route_bytes=T * D * b + D * N * b + T * N * 4 + T * K * 8 + (y_clear if by_router else 0),
        # x read once, its K copies written, the slot maps (+ the clear of y otherwise)
        permute_bytes=T * D * b + rows * D * b + T * K * 8 + (0 if by_router else y_clear),
        # the part of them that is written: x_perm (+ the clear of y when the permute does it)
        permute_write_bytes=rows * D * b + (0 if by_router else y_clear),
        combine_bytes=0 if fused_combine(wl, T) else rows * D * 4 + T * D * 4,
        up_weight_bytes=live * up_rows * D * b, down_weight_bytes=live * D * H * b,
        live_experts=live,
        # whole-layer bytes a memory-bound (decode) step must move: the live experts' weights, x, y, W_g
        decode_bytes=live * (up_rows * D + D * H) * b + T * D * b + T * D * 4 + D * N * b,
    )


def config_dict(wl, T, world):
    d = {"workload": wl.name, "T": T, "D": wl.D, "H": wl.H, "N": wl.N, "K": wl.K,
         "act": "swiglu" if wl.act == ACT_SWIGLU else "gelu", "global_batch": T * world,
         "parallelism": f"dp{world}", "l2": "flushed (512 MiB write) before every step"}
    if wl.n_shared:
        d["n_shared"] = wl.n_shared
    if wl.capacity_factor > 0:
        d["capacity_factor"] = wl.capacity_factor
        d["overflow"] = "reroute" if wl.overflow else "drop"
    return d


def fused_decode(wl, T):
    """Whether the library runs this layer as its one-kernel decode path: bf16, at most 64
    tokens and 32 experts, no shared expert, no reroute."""
    return (wl.dtype == torch.bfloat16 and 0 < T <= 64 and wl.N <= 32 and not wl.n_shared and
            not (wl.capacity_factor > 0 and wl.overflow))


def stream_floor_ms(nbytes, flush, dev, reps=10):
    """Median time of one plain read of nbytes from HBM (torch.sum over a bf16 tensor of that
    size, fp32 accumulation; L2 flushed before each run, CUDA events around the launch): what a
    single pass over that many bytes takes on this GPU, launch, ramp and tail included.  Context
    for a layer that must read the same bytes once (the decode path), not a bound it is held to."""
    t = torch.ones(max(nbytes // 2, 1), dtype=torch.bfloat16, device=dev)
    out = torch.empty((), dtype=torch.float32, device=dev)
    ms = []
    for i in range(reps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        torch.sum(t, dim=0, dtype=torch.float32, out=out)
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            ms.append(a.elapsed_time(b))
    del t
    return float(np.median(ms))


def write_floor_ms(nbytes, flush, dev, reps=8):
    """Median time of one plain write of nbytes to HBM (torch zero_ of a bf16 tensor that size;
    L2 flushed before each run, CUDA events around the launch).  On these B200s a write stream
    reaches well under the copy rate (which counts reads and writes), so it is the reference for a
    stage whose bytes are mostly written (the permute)."""
    t = torch.empty(max(nbytes // 2, 1), dtype=torch.bfloat16, device=dev)
    ms = []
    for i in range(reps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        t.zero_()
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            ms.append(a.elapsed_time(b))
    del t
    return float(np.median(ms))


def gemm_peak(pk, step_ms):
    """(peak TFLOP/s, its name): the sustained figure for kernels inside long steps, else the burst one."""
    if step_ms > SUSTAINED_STEP_MS and "bf16_tflops_sustained" in pk:
        return float(pk["bf16_tflops_sustained"]), "bf16 sustained"
    return float(pk["bf16_tflops"]), "bf16 burst"


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
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                pw.append(float(r[3]))
                for k, name in enumerate(names):
                    if r[5 + k].strip().lower() == "active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "power_w_max": max(pw) if pw else None, "samples": len(sm)}


# --------------------------------------------------------------------------- the oracle on the host cores
class OracleSample:
    """The fp64 oracle, as it stands, timed on a bounded sample of one workload's batch.

    Layers whose expert weights fit comfortably in host memory run the oracle's
    whole layer on a sample of tokens.  Larger layers (the DeepSeek shape, 22.5 GB
    of experts) run the oracle's router and gate on a sample of tokens, its expert
    FFN on a sample of (token, slot) pairs of a few experts (only those experts'
    weights are copied to the host) and its combine on the sampled tokens; the
    three per-unit times give the time of one whole token.  Tokens are
    independent, so both give tokens/s of the whole layer (extrapolated).
    """

    def __init__(self, wl, inp, seed=0, threads=None):
        import oracle

        self.oracle, self.wl = oracle, wl
        self.tag = oracle.F32 if wl.dtype == torch.float32 else oracle.BF16
        self.threads = threads or oracle.default_threads()
        self.T = inp["x"].shape[0]
        rng = np.random.default_rng(seed)
        self.order = rng.permutation(self.T)
        self.cur = 0
        h = lambda t: None if t is None else bf16_bits(t)  # noqa: E731
        self.x, self.Wg, self.bg = h(inp["x"]), h(inp["W_g"]), h(inp["b_g"])
        self.whole = expert_weight_bytes(wl) <= WHOLE_LAYER_WEIGHT_BYTES
        self.sec_tok = None
        if self.whole:
            self.W1, self.W2, self.b1, self.b2 = h(inp["W1"]), h(inp["W2"]), h(inp["b1"]), h(inp["b2"])
            return
        # untimed preparation: route a seeded sample of tokens with the oracle and keep
        # the (token, slot) pairs that fall on the m experts chosen most often among them
        R, m = min(self.T, 2048), 8
        rows = np.sort(self.order[:R])
        xr = self._load(rows)
        sc = self._scores(xr)
        sel = oracle.select_topk(sc, wl.K)
        cnt = np.bincount(sel.ravel(), minlength=wl.N)
        experts = [int(e) for e in np.argsort(-cnt, kind="stable")[:m] if cnt[e] > 0]
        self.pairs = [(i, int(sel[i, j])) for i in range(R) for j in range(wl.K) if int(sel[i, j]) in experts]
        self.pair_x = xr
        self.ew = {e: (h(inp["W1"][e]), h(inp["W2"][e]), None if inp["b1"] is None else h(inp["b1"][e]),
                       None if inp["b2"] is None else h(inp["b2"][e])) for e in experts}
        self.pcur = 0
        self.sec_r = self.sec_p = self.sec_c = None

    def _next_rows(self, n):
        idx = [self.order[(self.cur + i) % self.T] for i in range(n)]
        self.cur = (self.cur + n) % self.T
        return np.sort(np.array(idx, dtype=np.int64))

    def _load(self, rows):
        return self.oracle.load_rows(self.x, self.tag, rows)

    def _scores(self, xr):
        chunks = np.array_split(np.arange(xr.shape[0]), max(1, min(self.threads, xr.shape[0])))
        with ThreadPoolExecutor(len(chunks)) as ex:
            parts = list(ex.map(lambda c: self.oracle.router_scores(xr[c], self.Wg, self.tag, self.bg), chunks))
        return np.concatenate(parts)

    def step(self, budget_s):
        """One timed sample of about budget_s seconds.
        Returns (tokens/s of the whole layer, wall seconds of the sample, threads used, description)."""
        o, wl = self.oracle, self.wl
        if self.whole:
            n = self.threads if self.sec_tok is None else int(budget_s / self.sec_tok)
            n = max(1, min(self.T, n))
            rows = self._next_rows(n)
            xs = np.ascontiguousarray(self.x[rows])
            t0 = time.perf_counter()
            o.moe_layer(xs, self.Wg, self.W1, self.W2, K=wl.K, act=wl.act, dtype_tag=self.tag, bg=self.bg,
                        b1=self.b1, b2=self.b2, threads=self.threads)
            dt = time.perf_counter() - t0
            self.sec_tok = dt / n
            return n / dt, dt, min(self.threads, n), f"whole layer (router, top-k, experts, combine) on {n} of {self.T} tokens"
        K = wl.K
        if self.sec_r is None:
            n_r, n_p = 4 * self.threads, 2 * self.threads
        else:
            # split the budget as one token's time splits (router + K pairs + combine)
            tok = self.sec_r + K * self.sec_p + self.sec_c
            n_v = max(1.0, budget_s / tok)
            n_r = int(min(self.T, max(self.threads, n_v)))
            n_p = int(max(self.threads, n_v * K))
        rows = self._next_rows(n_r)
        pairs = [self.pairs[(self.pcur + i) % len(self.pairs)] for i in range(n_p)]
        self.pcur = (self.pcur + n_p) % len(self.pairs)
        t0 = time.perf_counter()
        xr = self._load(rows)
        sc = self._scores(xr)
        sel = o.select_topk(sc, K)
        w = o.gate_weights(sc, sel)
        t1 = time.perf_counter()

        def run(pair):
            i, e = pair
            W1e, W2e, b1e, b2e = self.ew[e]
            return o.expert(self.pair_x[i], wl.act, self.tag, W1e, W2e, b1e, b2e)

        with ThreadPoolExecutor(self.threads) as ex:
            E = list(ex.map(run, pairs))
        t2 = time.perf_counter()
        for i in range(n_r):
            o.combine(w[i], np.stack([E[(i * K + j) % n_p] for j in range(K)]))
        t3 = time.perf_counter()
        self.sec_r, self.sec_p, self.sec_c = (t1 - t0) / n_r, (t2 - t1) / n_p, (t3 - t2) / n_r
        tok = self.sec_r + K * self.sec_p + self.sec_c
        desc = (f"router + top-k + gate on {n_r} of {self.T} tokens, expert FFN on {n_p} (token, slot) pairs of "
                f"{len(self.ew)} experts, combine on {n_r} tokens; per-token time = router + {K} x pair + combine, "
                f"extrapolated to the whole layer")
        return 1.0 / tok, t3 - t0, self.threads, desc


def reference_inputs(wl):
    """The workload's inputs, drawn as the native arm draws them (on the GPU when there is one)."""
    if torch.cuda.is_available():
        return make_inputs(wl, "cuda", seed=wl.seed)
    return make_inputs(wl, "cpu", seed=wl.seed)


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    torch.manual_seed(0)
    inp = reference_inputs(wl)
    smp = OracleSample(wl, inp, seed=1)
    del inp
    if torch.cuda.is_available():
        torch.cuda.empty_cache()
    n = max(args.steps + args.warmup, 1)
    per_step = max(0.2, args.ref_seconds / n)
    rates, walls = [], []
    cores, sample = 1, ""
    for i in range(args.warmup + args.steps):
        r, wall, cores, sample = smp.step(per_step)
        if i >= args.warmup:
            rates.append(r)
            walls.append(wall)
    v = statistics.median(rates)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            # what one step actually ran (a bounded sample), not a whole layer
            "ms_per_step": 1000.0 * statistics.median(walls),
            "ms_per_layer_extrapolated": 1000.0 * wl.T / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(wl, wl.T, args.gpus), "extrapolated": True, "sample": sample,
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- native arm
def e2e_pipelined(moe, cfg, W, ws, wl, T, x_host, steps, warm, flush, dev, aux_bufs_fn, flush_each):
    """moe_forward through host buffers, copies overlapped with the neighbouring steps' kernels.

    Step i: copy-in of x on the h2d stream into x buffer i%2 (after forward i-2 has read it),
    forward on the compute stream (after its copy-in and after copy-out i-2 has read
    y / statistics buffer i%2), copy-out of y and the loss scalars on the d2h stream.
    Returns the milliseconds from the first copy-in to the last copy-out of the timed steps."""
    s_cmp = torch.cuda.current_stream(dev)
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xd = [torch.empty(x_host.shape, dtype=x_host.dtype, device=dev) for _ in range(2)]
    yd = [torch.empty(T, wl.D, dtype=torch.float32, device=dev) for _ in range(2)]
    yh = [torch.empty(T, wl.D, dtype=torch.float32).pin_memory() for _ in range(2)]
    sch = [torch.empty(4).pin_memory() for _ in range(2)]
    auxd = [aux_bufs_fn() for _ in range(2)]
    caux = [moe.make_aux(**a) for a in auxd]

    def run(n):
        ev_h2d = [torch.cuda.Event() for _ in range(n)]
        ev_fwd = [torch.cuda.Event() for _ in range(n)]
        ev_d2h = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_h2d)
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_h2d.wait_event(ev_fwd[i - 2])
            with torch.cuda.stream(s_h2d):
                xd[b].copy_(x_host, non_blocking=True)
            ev_h2d[i].record(s_h2d)
            s_cmp.wait_event(ev_h2d[i])
            if i >= 2:
                s_cmp.wait_event(ev_d2h[i - 2])
            if flush_each:
                flush.zero_()
            moe.check(moe.moe_forward(cfg, xd[b], T, W, yd[b], moe.MOE_F32, caux[b], ws, ws.numel(), s_cmp),
                      "e2e forward")
            ev_fwd[i].record(s_cmp)
            s_d2h.wait_event(ev_fwd[i])
            with torch.cuda.stream(s_d2h):
                yh[b].copy_(yd[b], non_blocking=True)
                sch[b].copy_(auxd[b]["scalars"], non_blocking=True)
            ev_d2h[i].record(s_d2h)
        t1.record(s_d2h)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    run(max(warm, 3))
    ms = run(steps)
    ok = torch.equal(yh[(steps - 1) % 2], yd[(steps - 1) % 2].cpu())
    return ms, ok


def backward_flops(wl, T):
    """FLOPs of the backward: the minimal chain rule (twice the forward's expert and router
    contractions) and the recomputed pre-activations on top."""
    c_up = 4 if wl.act == ACT_SWIGLU else 2
    minimal = 2 * (T * wl.K * (c_up + 2) * wl.D * wl.H + 2 * T * wl.D * wl.N)
    return minimal, minimal + T * wl.K * c_up * wl.D * wl.H


def run_backward(args, wl):
    """Time moe_backward (graph-captured, L2 flushed before every step) on one GPU."""
    import sparse_mixture_experts_10_b200 as moe
    from sparse_mixture_experts_10_b200 import build as moe_build

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    moe_build.build()
    moe.load_library()
    T = wl.T
    inp = make_inputs(wl, dev, seed=wl.seed)
    cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias)
    W = moe.make_weights(inp["W_g"], inp["W1"], inp["W2"], inp["b_g"], inp["b1"], inp["b2"], inp["b_sel"])
    rows1 = 2 * wl.H if wl.act == ACT_SWIGLU else wl.H
    dy = torch.randn(T, wl.D, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
    g = dict(dx=torch.empty(T, wl.D, device=dev), dW_g=torch.empty(wl.D, wl.N, device=dev),
             db_g=torch.empty(wl.N, device=dev), dW1=torch.empty(wl.N, rows1, wl.D, device=dev),
             dW2=torch.empty(wl.N, wl.D, wl.H, device=dev))
    if wl.has_bias:
        g["db1"] = torch.empty(wl.N, wl.H, device=dev)
        g["db2"] = torch.empty(wl.N, wl.D, device=dev)
    grads = moe.make_grads(**g)
    ws = torch.empty(moe.moe_backward_workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def step():
        moe.check(moe.moe_backward(cfg, inp["x"], T, W, dy, 0.01, 0.01, grads, ws, ws.numel()), "backward")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(0)
    sampler.start()
    for a, b in ev:
        flush.zero_()
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    st = moe.moe_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    minimal, with_recompute = backward_flops(wl, T)
    pk, pk_kind = peaks()
    # the contractions run on the CUDA cores in fp32: 148 SMs x 128 FMA lanes x 2 FLOP x the clock
    fp32_peak = 148 * 128 * 2 * float(pk.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
    line = {"metric": METRIC + " (backward pass)", "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": config_dict(wl, T, 1) | {"mode": "backward"},
            "tflops_minimal": minimal / (ms * 1e-3) / 1e12, "tflops_with_recompute": with_recompute / (ms * 1e-3) / 1e12,
            "roofline": {"bound": "alu", "unit": "TFLOP/s", "achieved": with_recompute / (ms * 1e-3) / 1e12,
                         "peak": fp32_peak, "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 x max SM clock",
                         "frac": with_recompute / (ms * 1e-3) / 1e12 / fp32_peak,
                         "frac_of_bf16_tensor": with_recompute / (ms * 1e-3) / 1e12 / float(pk["bf16_tflops"])},
            "clocks": clocks}
    print(json.dumps(line), flush=True)


def run_route(args, wl):
    """Time moe_route alone (graph-captured, L2 flushed before every step) on one GPU: scores,
    top-k, gate weights, statistics and dispatch tables, with only x and W_g allocated."""
    import sparse_mixture_experts_10_b200 as moe
    from sparse_mixture_experts_10_b200 import build as moe_build

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    moe_build.build()
    moe.load_library()
    T = wl.T
    gen = torch.Generator(device=dev).manual_seed(wl.seed)
    x = torch.randn(T, wl.D, device=dev, generator=gen).to(wl.dtype)
    Wg = (torch.randn(wl.D, wl.N, device=dev, generator=gen) * wl.w_std).to(wl.dtype)
    cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias)
    W = moe.make_weights(Wg, None, None)
    ws = moe.alloc_workspace(cfg, T)
    logits = torch.empty(T, wl.N, device=dev)
    idx = torch.empty(T, wl.K, dtype=torch.int32, device=dev)
    tw = torch.empty(T, wl.K, device=dev)
    counts = torch.empty(wl.N, dtype=torch.int32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def step():
        moe.check(moe.moe_route(cfg, x, T, W, logits, idx, tw, counts, ws, ws.numel()), "route")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(0)
    sampler.start()
    for a, b in ev:
        flush.zero_()
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    st = moe.moe_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    es = 2 if wl.dtype == torch.bfloat16 else 4
    # algorithmic bytes: x and W_g read, logits, top-k indices and weights written
    nbytes = T * wl.D * es + wl.D * wl.N * es + T * wl.N * 4 + T * wl.K * 8
    pk, pk_kind = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"metric": METRIC + " (routing stage)", "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": config_dict(wl, T, 1) | {"mode": "route"},
            "roofline": {"bound": "hbm", "unit": "GB/s", "achieved": gbs, "peak": float(pk["hbm_gbs"]),
                         "peak_kind": f"{pk_kind} copy", "frac": gbs / float(pk["hbm_gbs"]),
                         "bytes_per_step": nbytes},
            "clocks": clocks}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    wl = workload_from_args(args)
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if args.mode == "backward":
        run_backward(args, wl)
        return
    if args.mode == "route":
        run_route(args, wl)
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
    # data parallelism: the weights are the same on every rank, each rank draws its own tokens
    inp = make_inputs(wl, dev, seed=wl.seed)
    if rank > 0:
        gx = torch.Generator(device=dev).manual_seed(rank_seed(wl, rank))
        inp["x"] = torch.randn(T, wl.D, device=dev, generator=gx).to(wl.dtype)
    cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias, wl.n_shared,
                          wl.capacity_factor, wl.overflow)
    W = moe.make_weights(inp["W_g"], inp["W1"], inp["W2"], inp["b_g"], inp["b1"], inp["b2"], inp["b_sel"],
                         inp["S1"], inp["sb1"], inp["S2"], inp["sb2"])
    ws = moe.alloc_workspace(cfg, T)
    y = torch.empty(T, wl.D, dtype=torch.float32, device=dev)

    def aux_bufs():
        return dict(counts=torch.empty(wl.N, dtype=torch.int32, device=dev),
                    importance=torch.empty(wl.N, device=dev), p_mean=torch.empty(wl.N, device=dev),
                    scalars=torch.empty(4, device=dev))

    aux_t = aux_bufs()
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
    counts = aux_t["counts"].cpu().numpy()   # the router's choice, before any capacity
    kept = None
    if wl.capacity_factor > 0:   # the accepted pairs per expert, from the workspace tables
        Lw = moe.moe_get_workspace_layout(cfg, T)
        kept = ws[Lw.counts:Lw.counts + 4 * wl.N].view(torch.int32).cpu().numpy()

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

    gstats = GlobalStats(moe, cfg, wl, T, ws, dev) if world > 1 else None
    if gstats is not None:
        gstats.step()   # the collective's warm-up
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
        if gstats is not None:
            gstats.step()
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

    # ---- end to end through host buffers, copies overlapped with compute
    small = expert_weight_bytes(wl) + T * wl.D * 6 < 2 * (126 << 20)
    x_host = inp["x"].cpu().pin_memory()
    e2e_ms_local, e2e_ok = e2e_pipelined(moe, cfg, W, ws, wl, T, x_host, args.steps, args.warmup, flush, dev,
                                         aux_bufs, flush_each=small)
    e2e_ms = max_over_ranks(e2e_ms_local, dev, world)
    e2e_tps = job_throughput(T, world, args.steps, e2e_ms)
    h2d = T * wl.D * x_host.element_size()
    d2h = T * wl.D * 4 + 16

    # ---- global statistics over all ranks (data parallelism), as left by the last timed step
    aux_global = gstats.report() if gstats is not None else None

    # ---- roofline of the dominant kernel (its duration from the timed steps)
    wm = work_model(wl, T, counts, kept)
    pk, pk_kind = peaks()
    decode = wl.name.startswith("decode")
    if names[dom] in ("up", "down") and not decode:
        fl = wm["up_flops"] if names[dom] == "up" else wm["down_flops"]
        achieved = fl / (dom_mean_ms * 1e-3) / 1e12
        peak, peak_name = gemm_peak(pk, ms_per_step)
        roof = {"kernel": f"grouped_gemm_tc ({names[dom]})", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": f"{pk_kind} {peak_name}",
                "frac_of_burst": achieved / float(pk["bf16_tflops"]),
                "spec_peak": SPEC_PEAKS["bf16_tflops"], "frac_vs_spec": achieved / SPEC_PEAKS["bf16_tflops"]}
    else:
        byt = {"route": wm["route_bytes"], "permute": wm["permute_bytes"], "combine": wm["combine_bytes"],
               "up": wm["up_weight_bytes"], "down": wm["down_weight_bytes"]}.get(names[dom], 0)
        kname = names[dom]
        if fused_decode(wl, T) and names[dom] == "up":
            # the whole layer is one kernel between the "up" events: all of its bytes count
            byt, kname = wm["decode_bytes"], "decode_layer_kernel (whole layer, one launch)"
        achieved = byt / (dom_mean_ms * 1e-3) / 1e9
        peak = float(pk["hbm_gbs"])
        roof = {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"{pk_kind} copy",
                "spec_peak": SPEC_PEAKS["hbm_gbs"], "frac_vs_spec": achieved / SPEC_PEAKS["hbm_gbs"]}
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
            wb = int(wm["permute_write_bytes"])
            if not decode and wb >= (64 << 20) and mean_stage[s] > 0.02:
                # a plain write of the bytes the permute writes, timed the same way
                wf = write_floor_ms(wb, flush, dev)
                d["write_floor"] = {"ms": wf, "GB/s": wb / (wf * 1e-3) / 1e9, "bytes": wb,
                                    "how": "torch zero_ of a bf16 tensor of the permute's written bytes, L2 flushed, "
                                           "median of 8"}
                d["frac_of_write_floor"] = wf / mean_stage[s]
        elif nm == "combine":
            d["GB/s"] = wm["combine_bytes"] / (mean_stage[s] * 1e-3) / 1e9
        elif nm in ("up", "down"):
            fl = wm["up_flops"] if nm == "up" else wm["down_flops"]
            d["TFLOP/s"] = fl / (mean_stage[s] * 1e-3) / 1e12
            d["weight GB/s"] = (wm["up_weight_bytes"] if nm == "up" else wm["down_weight_bytes"]) / (
                mean_stage[s] * 1e-3) / 1e9
        stages[nm] = d

    # the layer as a whole: active FLOP rate, and for the expert GEMMs together
    layer = {"active_tflops": wm["flops"] / (ms_per_step * 1e-3) / 1e12}
    gemm_ms = float(mean_stage[names.index("up")] + mean_stage[names.index("down")])
    layer["gemm_tflops"] = (wm["up_flops"] + wm["down_flops"]) / (gemm_ms * 1e-3) / 1e12
    gp, gp_name = gemm_peak(pk, ms_per_step)
    layer["gemm_frac_vs_spec"] = layer["gemm_tflops"] / SPEC_PEAKS["bf16_tflops"]
    layer["gemm_frac_of_measured"] = layer["gemm_tflops"] / gp
    layer["active_frac_vs_spec"] = layer["active_tflops"] / SPEC_PEAKS["bf16_tflops"]
    if decode:
        gbs = wm["decode_bytes"] / (ms_per_step * 1e-3) / 1e9
        layer.update({"decode_bytes": wm["decode_bytes"], "GB/s": gbs, "frac_vs_spec": gbs / SPEC_PEAKS["hbm_gbs"],
                      "frac_of_measured": gbs / float(pk["hbm_gbs"]), "live_experts": wm["live_experts"]})
        # a plain read of the same bytes, timed the same way: the rate one pass of this size reaches
        fl_ms = stream_floor_ms(int(wm["decode_bytes"]), flush, dev)
        roof["stream_floor"] = {"ms": fl_ms, "GB/s": wm["decode_bytes"] / (fl_ms * 1e-3) / 1e9,
                                "frac_of_copy": wm["decode_bytes"] / (fl_ms * 1e-3) / 1e9 / float(pk["hbm_gbs"]),
                                "how": "torch.sum over a bf16 tensor of the layer's bytes, L2 flushed, median of 10"}
        roof["frac_of_stream_floor"] = fl_ms / dom_mean_ms

    line = {"metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
            "config": config_dict(wl, T, world),
            "active_tflops": wm["flops"] * world * args.steps / (total_ms / 1e3) / 1e12,
            "layer": layer, "roofline": roof, "stages": stages,
            "stages_note": f"{n_break} separate steps with an event between every two stages",
            "e2e": {"value": e2e_tps, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "overlap": "copy-in / copy-out on their own streams, double-buffered",
                    "l2": "flushed before every forward (inside the timed span)" if small
                    else "inputs and weights larger than L2", "y_copied_back_matches": bool(e2e_ok)},
            "gpu_launches": launches, "clocks": clocks}
    if aux_global is not None:
        line["aux_global"] = aux_global
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(wl, inp, seed=1)
        smp.step(min(2.0, args.cpu_seconds / 4))   # calibration
        v, _, cores, sample = smp.step(args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
                                "extrapolated": True}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


class GlobalStats:
    """The layer's statistics over the global batch under data parallelism: each rank's exact
    integer partial sums (moe_aux_partials, from the routing the layer left in its workspace)
    are all-reduced and finalised (moe_aux_finalize) identically on every rank."""

    def __init__(self, moe, cfg, wl, T, ws, dev):
        self.moe, self.cfg = moe, cfg
        L = moe.moe_get_workspace_layout(cfg, T)
        N, K = wl.N, wl.K
        view = lambda off, n, dt: ws[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)  # noqa: E731
        self.logits = view(L.logits, T * N, torch.float32)
        self.idx = view(L.topk_idx, T * K, torch.int32)
        self.w = view(L.topk_w, T * K, torch.float32)
        self.T = T
        self.part = torch.zeros(moe.aux_partials_len(N), dtype=torch.int64, device=dev)
        self.out = dict(counts=torch.empty(N, dtype=torch.int32, device=dev), importance=torch.empty(N, device=dev),
                        p_mean=torch.empty(N, device=dev), scalars=torch.empty(4, device=dev))
        self.caux = moe.make_aux(**self.out)

    def step(self):
        """Enqueue partials, the all-reduce (NCCL) and the finalisation on the current stream."""
        import torch.distributed as dist

        self.moe.check(self.moe.moe_aux_partials(self.cfg, self.T, self.logits, self.idx, self.w, self.part),
                       "partials")
        dist.all_reduce(self.part)
        self.moe.check(self.moe.moe_aux_finalize(self.cfg, self.part, self.caux), "finalize")

    def report(self):
        import torch.distributed as dist

        sc = self.out["scalars"].clone()
        lo, hi = sc.clone(), sc.clone()
        dist.all_reduce(lo, op=dist.ReduceOp.MIN)
        dist.all_reduce(hi, op=dist.ReduceOp.MAX)
        return {"tokens": int(self.part[-1].item()), "scalars": [float(v) for v in sc.tolist()],
                "identical_on_all_ranks": bool(torch.equal(lo, hi)),
                "in_timed_steps": "partials + all-reduce of 3N+1 int64 + finalise, every step"}


if __name__ == "__main__":
    main()
