"""fp64 oracle for the sparsely-gated MoE FFN layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``sparse_mixture_experts_10_b200``) never imports it, and this
package never imports the product.

The arithmetic lives in ``moe_oracle.c`` (plain fp64 loops, each function citing
the passage it follows).  This module only compiles that file with gcc,
marshals numpy arrays into it and runs disjoint token ranges on threads
(ctypes releases the GIL during each call, so the C code itself stays
single-threaded).

Array conventions: x and the weight matrices are either ``float32`` arrays or
``uint16`` arrays holding bf16 bit patterns (``dtype="bf16"``); the oracle widens
both exactly to double.  Biases are float32.

Parity notes: the smooth Load estimator of the Shazeer article is not
implemented (parity unpinned, out of scope); Load is the hard per-expert count.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

F32, BF16 = 0, 1
ACT_GELU, ACT_SWIGLU = 0, 1

_lib = None
_lock = threading.Lock()


def compile_source(src: str, out: str) -> str:
    """gcc -O2 without fast-math or FMA contraction, so every operation rounds as written."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-std=c11", "-Wall", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/_build/liboracle.so."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


class _Layer(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("x", ctypes.c_void_p), ("Wg", ctypes.c_void_p), ("bg", ctypes.c_void_p),
                ("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("bsel", ctypes.c_void_p),
                ("S1", ctypes.c_void_p), ("sb1", ctypes.c_void_p), ("S2", ctypes.c_void_p), ("sb2", ctypes.c_void_p)]


def configure(L):
    """Declare the C signatures on a loaded oracle library (also used on rebuilt copies in tests)."""
    i64, i32, vp, dp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
    L.orc_gelu.restype = dp
    L.orc_gelu.argtypes = [dp]
    L.orc_silu.restype = dp
    L.orc_silu.argtypes = [dp]
    L.orc_load_row.argtypes = [i64, vp, i32, i64, vp]
    L.orc_router_scores.argtypes = [i64, i64, vp, vp, i32, vp, vp]
    L.orc_expert_rank.restype = i64
    L.orc_expert_rank.argtypes = [i64, vp, i64]
    L.orc_rank_experts.argtypes = [i64, vp, vp]
    L.orc_select_topk.argtypes = [i64, i64, vp, vp]
    L.orc_softmax.argtypes = [i64, vp, vp]
    L.orc_gate_weights.argtypes = [i64, i64, vp, vp, vp]
    L.orc_expert_gelu.argtypes = [i64, i64, vp, vp, vp, vp, vp, i32, vp, vp]
    L.orc_expert_swiglu.argtypes = [i64, i64, vp, vp, vp, i32, vp, vp]
    L.orc_combine.argtypes = [i64, i64, vp, vp, vp]
    L.orc_add_shared.argtypes = [i64, vp, vp]
    L.orc_moe_layer_rows.argtypes = [ctypes.POINTER(_Layer), i64, i64, vp, vp, vp, vp, vp, vp, vp]
    L.orc_capacity_reroute.argtypes = [i64, i64, i64, vp, vp, i64, vp]
    L.orc_selection_values.argtypes = [ctypes.POINTER(_Layer), i64, i64, vp, vp, vp]
    L.orc_gelu_grad.restype = dp
    L.orc_gelu_grad.argtypes = [dp]
    L.orc_silu_grad.restype = dp
    L.orc_silu_grad.argtypes = [dp]
    L.orc_moe_layer_backward.argtypes = [ctypes.POINTER(_Layer), i64, vp, vp, dp, dp, vp, vp, vp, vp, vp, vp, vp]
    L.orc_capacity.restype = i64
    L.orc_capacity.argtypes = [dp, i64, i64, i64]
    L.orc_capacity_keep.argtypes = [i64, i64, i64, vp, i64, vp]
    L.orc_cv_squared.restype = dp
    L.orc_cv_squared.argtypes = [i64, vp]
    L.orc_simple_balance_loss.restype = dp
    L.orc_simple_balance_loss.argtypes = [i64, vp]
    L.orc_aux_stats.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp]
    for name in ("orc_expert_params", "orc_total_params", "orc_active_params"):
        getattr(L, name).restype = i64
    L.orc_expert_params.argtypes = [i64, i64, i32, i32]
    L.orc_total_params.argtypes = [i64, i64, i64, i64, i32, i32]
    L.orc_active_params.argtypes = [i64, i64, i64, i64, i32, i32]
    return L


def lib():
    """Load (building if needed) the oracle shared library."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = configure(ctypes.CDLL(build()))
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _mat(a, dtype_tag):
    """Contiguous copy in the storage dtype: float32, or uint16 for bf16 bits."""
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float32 if dtype_tag == F32 else np.uint16)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


# --- scalar helpers -------------------------------------------------------------------------------
def gelu(v: float) -> float:
    return lib().orc_gelu(float(v))


def silu(v: float) -> float:
    return lib().orc_silu(float(v))


# --- routing ----------------------------------------------------------------------------------------
def rank_experts(scores) -> np.ndarray:
    """The experts of one score row in rank order (descending score, equal scores: lower index first)."""
    s = _c(scores, np.float64)
    out = np.empty(s.shape[0], dtype=np.int32)
    lib().orc_rank_experts(s.shape[0], _p(s), _p(out))
    return out


def select_topk(scores, K: int) -> np.ndarray:
    """Top-K of each row of a [T, N] (or [N]) score array, best first."""
    s = np.atleast_2d(_c(scores, np.float64))
    T, N = s.shape
    out = np.empty((T, K), dtype=np.int32)
    L = lib()
    for t in range(T):
        L.orc_select_topk(N, K, _p(s[t]), _p(out[t]))
    return out


def gate_weights(scores, sel) -> np.ndarray:
    """Slot weights G(x)[sel_j] of G = softmax(KeepTopK(scores)) with the kept set sel, per row."""
    s = np.atleast_2d(_c(scores, np.float64))
    sl = np.atleast_2d(_c(sel, np.int32))
    T, K = sl.shape
    N = s.shape[1]
    out = np.empty((T, K), dtype=np.float64)
    L = lib()
    for t in range(T):
        L.orc_gate_weights(N, K, _p(s[t]), _p(sl[t]), _p(out[t]))
    return out


def softmax(v) -> np.ndarray:
    """softmax of one vector (entries of -inf get probability 0)."""
    a = _c(v, np.float64)
    out = np.empty_like(a)
    lib().orc_softmax(a.shape[0], _p(a), _p(out))
    return out


def load_rows(x, dtype_tag, rows) -> np.ndarray:
    """Widen the given token rows of x to fp64 [len(rows), D]."""
    xm = _mat(x, dtype_tag)
    D = xm.shape[-1]
    out = np.empty((len(rows), D), dtype=np.float64)
    L = lib()
    for i, t in enumerate(rows):
        L.orc_load_row(D, _p(xm), dtype_tag, int(t), _p(out[i]))
    return out


def router_scores(x_rows64, Wg, dtype_tag, bg=None) -> np.ndarray:
    """fp64 scores for fp64 token rows [R, D] against W_g [D, N]."""
    xr = np.atleast_2d(_c(x_rows64, np.float64))
    W = _mat(Wg, dtype_tag)
    b = _c(bg, np.float32)
    R, D = xr.shape
    N = W.shape[1]
    out = np.empty((R, N), dtype=np.float64)
    L = lib()
    for r in range(R):
        L.orc_router_scores(D, N, _p(xr[r]), _p(W), dtype_tag, _p(b), _p(out[r]))
    return out


# --- experts and combine ----------------------------------------------------------------------------
def expert(x_row64, act, dtype_tag, W1e, W2e, b1e=None, b2e=None, return_hidden=False):
    """One expert's output for one fp64 token row. W1e: [H, D] (GELU) or [2H, D] (SwiGLU); W2e: [D, H].
    With return_hidden, also the hidden activations [H] (after GELU, or silu(gate) * up)."""
    xr = _c(x_row64, np.float64)
    A = _mat(W1e, dtype_tag)
    B = _mat(W2e, dtype_tag)
    D, H = B.shape
    hid = np.empty(H, dtype=np.float64)
    out = np.empty(D, dtype=np.float64)
    L = lib()
    if act == ACT_GELU:
        L.orc_expert_gelu(D, H, _p(xr), _p(A), _p(_c(b1e, np.float32)), _p(B), _p(_c(b2e, np.float32)),
                          dtype_tag, _p(hid), _p(out))
    else:
        L.orc_expert_swiglu(D, H, _p(xr), _p(A), _p(B), dtype_tag, _p(hid), _p(out))
    return (out, hid) if return_hidden else out


def combine(w, E) -> np.ndarray:
    """y = sum_j w_j E_j in slot order for one token: w [K], E [K, D]."""
    wv = _c(w, np.float64)
    Em = _c(E, np.float64)
    K, D = Em.shape
    y = np.empty(D, dtype=np.float64)
    lib().orc_combine(K, D, _p(wv), _p(Em), _p(y))
    return y


def add_shared(y, s) -> np.ndarray:
    """y + s (the shared expert's output added after the routed sum), one token."""
    yv = np.array(_c(y, np.float64))
    sv = _c(s, np.float64)
    lib().orc_add_shared(yv.shape[0], _p(sv), _p(yv))
    return yv


def capacity(cf: float, T: int, K: int, N: int) -> int:
    """Per-expert capacity ceil(cf T K / N); no limit (a huge number) for cf <= 0."""
    return lib().orc_capacity(float(cf), T, K, N)


def capacity_keep(sel, N: int, C: int) -> np.ndarray:
    """Drop decisions [T, K] (1 kept, 0 dropped): rows served in order, C per expert."""
    sl = np.ascontiguousarray(np.atleast_2d(sel), dtype=np.int32)
    T, K = sl.shape
    keep = np.zeros((T, K), dtype=np.uint8)
    lib().orc_capacity_keep(T, N, K, _p(sl), int(C), _p(keep))
    return keep


def moe_layer(x, Wg, W1, W2, *, K, act, dtype_tag, bg=None, b1=None, b2=None, sel_scores=None,
              threads=None, rows=None, bsel=None, S1=None, S2=None, sb1=None, sb2=None, keep=None, assign=None):
    """The whole layer on host arrays, in fp64.

    x [T, D]; Wg [D, N]; W1 [N, H, D] (GELU) or [N, 2H, D] (SwiGLU); W2 [N, D, H].
    bsel [N] float32 (optional): selection-only bias (changes the kept set, not the weights).
    S1 [H or 2H, D], S2 [D, H], sb1 [H], sb2 [D] (optional): the shared expert.
    sel_scores [T, N] float32 (optional): make the expert selection on these scores
    (the device's fp32 logits, plus any selection bias in fp32) while the gate
    weights use the fp64 scores.
    keep [T, K] uint8 (optional): capacity decisions (capacity_keep); dropped slots add nothing.
    assign [T, K] int32 (optional): the expert serving each slot after a reroute
    (capacity_reroute), -1 for none; each slot keeps its gate weight.
    rows: optional (t0, t1) range; other rows of the outputs are left as zeros.
    Returns dict(scores [T,N], sel [T,K], w [T,K], y [T,D]) in fp64 / int32.
    """
    xm = _mat(x, dtype_tag)
    T, D = xm.shape
    Wgm = _mat(Wg, dtype_tag)
    N = Wgm.shape[1]
    W2m = _mat(W2, dtype_tag)
    H = W2m.shape[2]
    W1m = _mat(W1, dtype_tag)
    bgm, b1m, b2m = _c(bg, np.float32), _c(b1, np.float32), _c(b2, np.float32)
    ss = _c(sel_scores, np.float32)
    kp = _c(keep, np.uint8)
    asg = _c(assign, np.int32)
    bselm, S1m, S2m = _c(bsel, np.float32), _mat(S1, dtype_tag), _mat(S2, dtype_tag)
    sb1m, sb2m = _c(sb1, np.float32), _c(sb2, np.float32)
    lay = _Layer(D, H, N, K, act, dtype_tag, _p(xm), _p(Wgm), _p(bgm), _p(W1m), _p(b1m), _p(W2m), _p(b2m),
                 _p(bselm), _p(S1m), _p(sb1m), _p(S2m), _p(sb2m))
    scores = np.zeros((T, N), dtype=np.float64)
    sel = np.zeros((T, K), dtype=np.int32)
    w = np.zeros((T, K), dtype=np.float64)
    y = np.zeros((T, D), dtype=np.float64)
    t0, t1 = rows if rows is not None else (0, T)
    nthr = threads or default_threads()
    L = lib()
    if t1 <= t0:
        return dict(scores=scores, sel=sel, w=w, y=y)
    step = max(1, -(-(t1 - t0) // (nthr * 4)))
    ranges = [(a, min(a + step, t1)) for a in range(t0, t1, step)]

    def run(r):
        L.orc_moe_layer_rows(ctypes.byref(lay), r[0], r[1], _p(ss), _p(kp), _p(asg), _p(scores), _p(sel), _p(w), _p(y))

    if nthr == 1 or len(ranges) == 1:
        for r in ranges:
            run(r)
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(run, ranges))
    return dict(scores=scores, sel=sel, w=w, y=y)


def selection_values(scores, bsel=None, sel_scores=None) -> np.ndarray:
    """The values experts are ranked on for selection, [T, N] fp64: the given fp32
    selection scores, else the fp64 scores plus the selection-only bias."""
    sc = np.ascontiguousarray(scores, dtype=np.float64)
    T, N = sc.shape
    bs, ss = _c(bsel, np.float32), _c(sel_scores, np.float32)
    lay = _Layer(0, 0, N, 0, 0, 0, None, None, None, None, None, None, None, _p(bs), None, None, None, None)
    v = np.zeros((T, N), dtype=np.float64)
    lib().orc_selection_values(ctypes.byref(lay), 0, T, _p(sc), _p(ss), _p(v))
    return v


def capacity_reroute(v, sel, C: int) -> np.ndarray:
    """Reroute decisions [T, K] int32: the expert serving each slot (-1: dropped)."""
    vv = np.ascontiguousarray(v, dtype=np.float64)
    sl = np.ascontiguousarray(sel, dtype=np.int32)
    T, K = sl.shape
    N = vv.shape[1]
    assign = np.zeros((T, K), dtype=np.int32)
    lib().orc_capacity_reroute(T, N, K, _p(vv), _p(sl), int(C), _p(assign))
    return assign


def moe_layer_capacity(x, Wg, W1, W2, *, K, act, dtype_tag, cf, sel_scores=None, overflow="drop", **kw):
    """The layer with a per-expert capacity: route every token, decide which
    assignments fit (rows in order, C = capacity(cf, T, K, N) each) and what
    happens to the others (overflow "drop" or "reroute"), then evaluate."""
    routed = moe_layer(x, Wg, np.zeros_like(W1), np.zeros_like(W2), K=K, act=act, dtype_tag=dtype_tag,
                       sel_scores=sel_scores, **{k: v for k, v in kw.items() if k in ("bg", "bsel", "threads")})
    T = routed["sel"].shape[0]
    N = _mat(Wg, dtype_tag).shape[1]
    C = capacity(cf, T, K, N)
    if overflow == "drop":
        keep = capacity_keep(routed["sel"], N, C)
        out = moe_layer(x, Wg, W1, W2, K=K, act=act, dtype_tag=dtype_tag, sel_scores=sel_scores, keep=keep, **kw)
        out["keep"] = keep
    elif overflow == "reroute":
        v = selection_values(routed["scores"], kw.get("bsel"), sel_scores)
        assign = capacity_reroute(v, routed["sel"], C)
        out = moe_layer(x, Wg, W1, W2, K=K, act=act, dtype_tag=dtype_tag, sel_scores=sel_scores, assign=assign,
                        **kw)
        out["assign"], out["keep"] = assign, (assign >= 0).astype(np.uint8)
    else:
        raise ValueError(f"overflow must be 'drop' or 'reroute', not {overflow!r}")
    out["capacity"] = C
    return out


def moe_layer_backward(x, Wg, W1, W2, dy, *, K, act, dtype_tag, bg=None, b1=None, b2=None, bsel=None,
                       sel_scores=None, alpha_switch=0.0, alpha_importance=0.0):
    """Gradients of sum(y * dy) + alpha_switch * switch_loss + alpha_importance * cv2_importance
    with respect to x, W_g, b_g, W1, b1, W2, b2 (fp64, single thread).  Returns a dict."""
    xm = _mat(x, dtype_tag)
    T, D = xm.shape
    Wgm = _mat(Wg, dtype_tag)
    N = Wgm.shape[1]
    W1m, W2m = _mat(W1, dtype_tag), _mat(W2, dtype_tag)
    H = W2m.shape[2]
    bgm, b1m, b2m, bselm = _c(bg, np.float32), _c(b1, np.float32), _c(b2, np.float32), _c(bsel, np.float32)
    ss = _c(sel_scores, np.float32)
    dyv = _c(dy, np.float64)
    lay = _Layer(D, H, N, K, act, dtype_tag, _p(xm), _p(Wgm), _p(bgm), _p(W1m), _p(b1m), _p(W2m), _p(b2m),
                 _p(bselm), None, None, None, None)
    out = dict(dx=np.empty((T, D)), dWg=np.empty((D, N)), dbg=np.empty(N), dW1=np.empty(W1m.shape),
               dW2=np.empty(W2m.shape))
    out["db1"] = np.empty((N, H)) if act == ACT_GELU else None
    out["db2"] = np.empty((N, D)) if act == ACT_GELU else None
    lib().orc_moe_layer_backward(ctypes.byref(lay), T, _p(ss), _p(dyv), float(alpha_switch), float(alpha_importance),
                                 _p(out["dx"]), _p(out["dWg"]), _p(out["dbg"]), _p(out["dW1"]), _p(out["db1"]),
                                 _p(out["dW2"]), _p(out["db2"]))
    return out


# --- statistics ---------------------------------------------------------------------------------------
def cv_squared(v) -> float:
    a = _c(v, np.float64)
    return lib().orc_cv_squared(a.shape[0], _p(a))


def simple_balance_loss(counts) -> float:
    a = _c(counts, np.float64)
    return lib().orc_simple_balance_loss(a.shape[0], _p(a))


def aux_stats(scores, sel, w, N: int):
    """counts, importance, p_mean [N] and scalars [switch, simple, cv2_importance, cv2_load]."""
    s = np.atleast_2d(_c(scores, np.float64)).reshape(-1, N)
    T = s.shape[0]
    sl = np.atleast_2d(_c(sel, np.int32))
    K = sl.shape[1]
    sl = sl.reshape(T, K)
    wv = _c(w, np.float64).reshape(T, K)
    counts = np.empty(N)
    imp = np.empty(N)
    pm = np.empty(N)
    sc = np.empty(4)
    lib().orc_aux_stats(T, N, K, _p(s), _p(sl), _p(wv), _p(counts), _p(imp), _p(pm), _p(sc))
    return dict(counts=counts, importance=imp, p_mean=pm, switch=sc[0], simple=sc[1],
                cv2_importance=sc[2], cv2_load=sc[3])


# --- parameter accounting -------------------------------------------------------------------------------
def expert_params(D, H, act=ACT_GELU, has_bias=False) -> int:
    return lib().orc_expert_params(D, H, act, int(bool(has_bias)))


def total_params(D, H, N, K, act=ACT_GELU, has_bias=False) -> int:
    return lib().orc_total_params(D, H, N, K, act, int(bool(has_bias)))


def active_params(D, H, N, K, act=ACT_GELU, has_bias=False) -> int:
    return lib().orc_active_params(D, H, N, K, act, int(bool(has_bias)))
