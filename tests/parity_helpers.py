"""Oracle-side helpers for the GPU parity tests.

The fp64 oracle is evaluated on host copies of exactly the inputs the device
saw.  For the full-size workloads only sampled token rows are evaluated, and
each expert's weights are copied to the host only when a sampled row uses it.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from moe_inputs import bf16_bits

# tolerances (stated once, used by every parity test)
LOGIT_RTOL = 1e-4          # |l_gpu - l_ref| <= 1e-4 * max_e |l_ref[t, e]|  (row-scaled)
BF16_MAX_ABS = 2e-2        # bf16 layer outputs vs fp64
BF16_REL_L2 = 1e-2
F32_REL = 1e-4             # fp32 layer outputs: max-abs <= 1e-4 * max|y_ref| and rel-L2 <= 1e-4


def tag(dtype: torch.dtype) -> int:
    return oracle.F32 if dtype == torch.float32 else oracle.BF16


def host(t):
    return None if t is None else bf16_bits(t)


def assert_logits_close(l_gpu: np.ndarray, l_ref: np.ndarray):
    scale = np.maximum(np.abs(l_ref).max(axis=1, keepdims=True), 1e-30)
    err = np.abs(l_gpu.astype(np.float64) - l_ref) / scale
    assert err.max() <= LOGIT_RTOL, f"logit error {err.max():.3e} (row-scaled) > {LOGIT_RTOL}"
    return float(err.max())


def assert_weights_close(w_gpu: np.ndarray, w_ref: np.ndarray, l_ref: np.ndarray):
    # the softmax moves by at most about twice the logit error, which is bounded row-wise above
    bound = 2 * LOGIT_RTOL * np.abs(l_ref).max(axis=1, keepdims=True) + 1e-6
    err = np.abs(w_gpu.astype(np.float64) - w_ref)
    assert np.all(err <= bound), f"gate weight error {err.max():.3e}"


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, dtype: torch.dtype):
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300))
    if dtype == torch.float32:
        assert max_abs <= F32_REL * max(float(np.abs(y_ref).max()), 1e-30), f"max-abs {max_abs:.3e}"
        assert rel_l2 <= F32_REL, f"rel-L2 {rel_l2:.3e}"
    else:
        assert max_abs <= BF16_MAX_ABS, f"max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
        assert rel_l2 <= BF16_REL_L2, f"rel-L2 {rel_l2:.3e} > {BF16_REL_L2}"
    return max_abs, rel_l2


def selection_scores(logits, inp):
    """What the device ranks: its fp32 logits, plus the selection-only bias added in fp32."""
    lg = np.asarray(logits, dtype=np.float32)
    b = inp.get("b_sel")
    return lg if b is None else (lg + host(b).astype(np.float32)).astype(np.float32)


def shared_kwargs(inp):
    return dict(S1=host(inp.get("S1")), S2=host(inp.get("S2")), sb1=host(inp.get("sb1")), sb2=host(inp.get("sb2")))


def capacity_factor(wl) -> float:
    """The capacity factor as the library receives it (an fp32 field), widened to double."""
    return float(np.float32(wl.capacity_factor))


def oracle_full_layer(inp, wl, K, gpu_logits=None, threads=None):
    """The whole layer on every token (small workloads); with the workload's capacity when it has one."""
    t = tag(wl.dtype)
    sel = None if gpu_logits is None else selection_scores(gpu_logits, inp)
    args = (host(inp["x"]), host(inp["W_g"]), host(inp["W1"]), host(inp["W2"]))
    kw = dict(K=K, act=wl.act, dtype_tag=t, bg=host(inp["b_g"]), b1=host(inp["b1"]), b2=host(inp["b2"]),
              sel_scores=sel, threads=threads, bsel=host(inp.get("b_sel")), **shared_kwargs(inp))
    if wl.capacity_factor > 0:
        return oracle.moe_layer_capacity(*args, cf=capacity_factor(wl),
                                         overflow="reroute" if wl.overflow else "drop", **kw)
    return oracle.moe_layer(*args, **kw)


def oracle_rows(inp, wl, K, rows, gpu_logits, threads=None):
    """Oracle results for the given token rows only, selecting on the device's fp32 logits.

    Returns dict(scores [R,N], sel [R,K], w [R,K], y [R,D]) in fp64 / int32."""
    t = tag(wl.dtype)
    rows = np.asarray(rows, dtype=np.int64)
    xr = oracle.load_rows(host(inp["x"][rows]), t, range(len(rows)))
    scores = oracle.router_scores(xr, host(inp["W_g"]), t, host(inp["b_g"]))
    sel = oracle.select_topk(selection_scores(gpu_logits[rows], inp).astype(np.float64), K)
    w = oracle.gate_weights(scores, sel)
    D = wl.D
    E = np.zeros((len(rows), K, D), dtype=np.float64)
    jobs = {}
    for i in range(len(rows)):
        for j in range(K):
            jobs.setdefault(int(sel[i, j]), []).append((i, j))
    nthr = threads or oracle.default_threads()
    with ThreadPoolExecutor(nthr) as ex:
        for e, pairs in sorted(jobs.items()):
            W1e = host(inp["W1"][e])
            W2e = host(inp["W2"][e])
            b1e = None if inp["b1"] is None else host(inp["b1"][e])
            b2e = None if inp["b2"] is None else host(inp["b2"][e])

            def run(pair, W1e=W1e, W2e=W2e, b1e=b1e, b2e=b2e):
                i, j = pair
                E[i, j] = oracle.expert(xr[i], wl.act, t, W1e, W2e, b1e, b2e)

            list(ex.map(run, pairs))
    y = np.stack([oracle.combine(w[i], E[i]) for i in range(len(rows))]) if len(rows) else np.zeros((0, D))
    if inp.get("S1") is not None:
        sk = shared_kwargs(inp)

        def shared(i):
            return oracle.add_shared(y[i], oracle.expert(xr[i], wl.act, t, sk["S1"], sk["S2"], sk["sb1"], sk["sb2"]))

        with ThreadPoolExecutor(nthr) as ex:
            y = np.stack(list(ex.map(shared, range(len(rows))))) if len(rows) else y
    return dict(scores=scores, sel=sel, w=w, y=y)


def sample_rows(T, n, gpu_idx, N, seed=0, least_loaded=2):
    """n seeded random rows plus every row of the `least_loaded` least-loaded non-empty experts,
    and the first and last row."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(T, size=min(n, T), replace=False).tolist()) | {0, T - 1}
    counts = np.bincount(gpu_idx.ravel(), minlength=N)
    nonempty = [e for e in np.argsort(counts, kind="stable") if counts[e] > 0][:least_loaded]
    for e in nonempty:
        rows |= set(np.nonzero((gpu_idx == e).any(axis=1))[0][:64].tolist())
    return np.array(sorted(rows), dtype=np.int64)


def expert_end_rows(gpu_idx, N):
    """For every expert with tokens, the first and the last token routed to it (the rows that
    open and close its segment of the permuted buffers)."""
    T, K = gpu_idx.shape
    rows = set()
    for e in range(N):
        toks = np.nonzero((gpu_idx == e).any(axis=1))[0]
        if toks.size:
            rows |= {int(toks[0]), int(toks[-1])}
    return np.array(sorted(rows), dtype=np.int64)


def oracle_scores(inp, wl, rows, threads=None):
    """fp64 router scores of the given token rows, computed on host threads."""
    t = tag(wl.dtype)
    rows = np.asarray(rows, dtype=np.int64)
    xr = oracle.load_rows(host(inp["x"][torch.from_numpy(rows).to(inp["x"].device)]), t, range(len(rows)))
    Wg, bg = host(inp["W_g"]), host(inp["b_g"])
    nthr = threads or oracle.default_threads()
    chunks = [c for c in np.array_split(np.arange(len(rows)), nthr) if c.size]
    with ThreadPoolExecutor(len(chunks)) as ex:
        parts = list(ex.map(lambda c: oracle.router_scores(xr[c], Wg, t, bg), chunks))
    return np.concatenate(parts)
