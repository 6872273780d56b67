"""Sparsely-gated Mixture-of-Experts FFN layer for one NVIDIA B200 (sm_100a).

This package is a thin ctypes binding of ``libmoe.so``, whose C ABI is declared
in ``include/moe.h``.  The functions here carry the same names and arguments as
the C entry points and only marshal arguments: torch tensors become device
pointers, streams become ``cudaStream_t`` handles.  Every step of the layer runs
in the library's CUDA kernels; there is no Python or CPU fallback, and importing
the package fails loudly when the library has not been built
(``python -m sparse_mixture_experts_10_b200.build``).

PyTorch is used only to hold device memory and to name streams.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_BOUNDS_CHECK=1 selects the bounds-check build of the same library (build.py --bounds-check)
LIB_PATH = os.path.join(_PKG, "libmoe_debug.so" if os.environ.get("MOE_BOUNDS_CHECK") == "1" else "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_GELU, MOE_ACT_SWIGLU = 0, 1
MOE_OVERFLOW_DROP, MOE_OVERFLOW_REROUTE = 0, 1
MOE_N_STAGES = 7
STAGE_NAMES = ("route", "scan", "permute", "up", "down", "combine", "stats")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_WORKSPACE_TOO_SMALL = -2
MOE_ERR_UNSUPPORTED = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_DEVICE_BOUNDS = -6
MOE_STATUS_TIMEOUT, MOE_STATUS_BOUNDS, MOE_STATUS_NAN_LOGIT = 1, 2, 4
MOE_NOALLOC_SCRATCH_BYTES = 2 << 20

EXPORTED = ("moe_workspace_size", "moe_route", "moe_forward", "moe_forward_timed", "moe_aux_stats",
            "moe_aux_stats_noalloc", "moe_aux_partials", "moe_aux_finalize", "moe_aux_finalize_host",
            "moe_ep_workspace_size", "moe_ep_dispatch", "moe_ep_experts_workspace_size", "moe_ep_experts",
            "moe_ep_combine", "moe_backward_workspace_size", "moe_backward",
            "moe_get_workspace_layout", "moe_total_params", "moe_active_params", "moe_get_device_status",
            "moe_launch_count", "moe_error_string", "moe_selftest_wait_timeout")


class moe_config(ctypes.Structure):
    _fields_ = [("DModel", ctypes.c_int32), ("DHidden", ctypes.c_int32), ("NExperts", ctypes.c_int32),
                ("TopK", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("has_bias", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
                ("overflow", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [("W_g", ctypes.c_void_p), ("b_g", ctypes.c_void_p), ("W1", ctypes.c_void_p),
                ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
                ("b_sel", ctypes.c_void_p), ("S1", ctypes.c_void_p), ("sb1", ctypes.c_void_p),
                ("S2", ctypes.c_void_p), ("sb2", ctypes.c_void_p)]


class moe_aux(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("importance", ctypes.c_void_p), ("p_mean", ctypes.c_void_p),
                ("scalars", ctypes.c_void_p)]


class moe_grads(ctypes.Structure):
    _fields_ = [("dx", ctypes.c_void_p), ("dW_g", ctypes.c_void_p), ("db_g", ctypes.c_void_p),
                ("dW1", ctypes.c_void_p), ("db1", ctypes.c_void_p), ("dW2", ctypes.c_void_p), ("db2", ctypes.c_void_p)]


class moe_workspace_layout(ctypes.Structure):
    _fields_ = [("total", ctypes.c_size_t), ("logits", ctypes.c_size_t), ("topk_idx", ctypes.c_size_t),
                ("topk_w", ctypes.c_size_t), ("counts", ctypes.c_size_t), ("offsets", ctypes.c_size_t),
                ("row_offsets", ctypes.c_size_t), ("perm_slot", ctypes.c_size_t), ("slot_row", ctypes.c_size_t),
                ("x_perm", ctypes.c_size_t), ("h", ctypes.c_size_t), ("z", ctypes.c_size_t),
                ("rows_cap", ctypes.c_int64), ("row_align", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} ({code})" if what else f"{error_string(code)} ({code})")


_lib = None


def load_library():
    """Load libmoe.so and declare its signatures.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_mixture_experts_10_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(moe_config)
    wp = ctypes.POINTER(moe_weights)
    auxp = ctypes.POINTER(moe_aux)
    L.moe_workspace_size.restype = sz
    L.moe_workspace_size.argtypes = [cfgp, i64]
    L.moe_route.restype = ctypes.c_int
    L.moe_route.argtypes = [cfgp, vp, i64, wp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_forward.restype = ctypes.c_int
    L.moe_forward.argtypes = [cfgp, vp, i64, wp, vp, i32, auxp, vp, sz, vp]
    L.moe_forward_timed.restype = ctypes.c_int
    L.moe_forward_timed.argtypes = [cfgp, vp, i64, wp, vp, i32, auxp, vp, sz, vp, ctypes.POINTER(vp)]
    L.moe_aux_stats.restype = ctypes.c_int
    L.moe_aux_stats.argtypes = [cfgp, i64, vp, vp, vp, auxp, vp, sz, vp]
    L.moe_aux_stats_noalloc.restype = ctypes.c_int
    L.moe_aux_stats_noalloc.argtypes = [cfgp, i64, vp, vp, vp, auxp, vp]
    L.moe_aux_partials.restype = ctypes.c_int
    L.moe_aux_partials.argtypes = [cfgp, i64, vp, vp, vp, vp, vp]
    L.moe_aux_finalize.restype = ctypes.c_int
    L.moe_aux_finalize.argtypes = [cfgp, vp, auxp, vp]
    L.moe_aux_finalize_host.restype = ctypes.c_int
    L.moe_aux_finalize_host.argtypes = [cfgp, vp, vp, vp, vp, vp]
    L.moe_ep_workspace_size.restype = sz
    L.moe_ep_workspace_size.argtypes = [cfgp, i32, i64]
    L.moe_ep_dispatch.restype = ctypes.c_int
    L.moe_ep_dispatch.argtypes = [cfgp, i32, vp, i64, wp, vp, vp, vp, vp, vp, auxp, vp, sz, vp]
    L.moe_ep_experts_workspace_size.restype = sz
    L.moe_ep_experts_workspace_size.argtypes = [cfgp, i64]
    L.moe_ep_experts.restype = ctypes.c_int
    L.moe_ep_experts.argtypes = [cfgp, vp, i64, vp, vp, wp, vp, vp, sz, vp]
    L.moe_ep_combine.restype = ctypes.c_int
    L.moe_ep_combine.argtypes = [cfgp, vp, i64, vp, vp, i32, vp]
    L.moe_backward_workspace_size.restype = sz
    L.moe_backward_workspace_size.argtypes = [cfgp, i64]
    L.moe_backward.restype = ctypes.c_int
    L.moe_backward.argtypes = [cfgp, vp, i64, wp, vp, ctypes.c_float, ctypes.c_float, ctypes.POINTER(moe_grads), vp,
                               sz, vp]
    L.moe_get_workspace_layout.restype = ctypes.c_int
    L.moe_get_workspace_layout.argtypes = [cfgp, i64, ctypes.POINTER(moe_workspace_layout)]
    L.moe_total_params.restype = i64
    L.moe_total_params.argtypes = [cfgp]
    L.moe_active_params.restype = i64
    L.moe_active_params.argtypes = [cfgp]
    L.moe_get_device_status.restype = ctypes.c_int
    L.moe_get_device_status.argtypes = []
    L.moe_launch_count.restype = i64
    L.moe_launch_count.argtypes = []
    L.moe_error_string.restype = ctypes.c_char_p
    L.moe_error_string.argtypes = [ctypes.c_int]
    L.moe_selftest_wait_timeout.restype = ctypes.c_int
    L.moe_selftest_wait_timeout.argtypes = [i64, vp]
    _lib = L
    return L


# ------------------------------------------------------------------ marshalling helpers
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return MOE_F32
    if dt == torch.bfloat16:
        return MOE_BF16
    raise ValueError(f"unsupported dtype {dt}")


def make_config(DModel, DHidden, NExperts, TopK, act=MOE_ACT_GELU, dtype=MOE_BF16, has_bias=False,
                n_shared=0, capacity_factor=0.0, overflow=MOE_OVERFLOW_DROP) -> moe_config:
    return moe_config(DModel, DHidden, NExperts, TopK, act, dtype, int(bool(has_bias)), int(n_shared),
                      float(capacity_factor), int(overflow))


def make_weights(W_g, W1, W2, b_g=None, b1=None, b2=None, b_sel=None, S1=None, sb1=None, S2=None,
                 sb2=None) -> moe_weights:
    return moe_weights(_ptr(W_g), _ptr(b_g), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(b_sel), _ptr(S1),
                       _ptr(sb1), _ptr(S2), _ptr(sb2))


def make_aux(counts=None, importance=None, p_mean=None, scalars=None) -> moe_aux:
    return moe_aux(_ptr(counts), _ptr(importance), _ptr(p_mean), _ptr(scalars))


def check(rc: int, what: str = "") -> int:
    if rc != MOE_OK:
        raise MoeError(rc, what)
    return rc


def error_string(code: int) -> str:
    return load_library().moe_error_string(code).decode()


# ------------------------------------------------------------------ the C entry points
def moe_workspace_size(cfg: moe_config, T: int) -> int:
    return load_library().moe_workspace_size(ctypes.byref(cfg), T)


def moe_route(cfg, x, T, weights, logits, topk_idx, topk_w, counts, ws, ws_bytes, stream=None) -> int:
    return load_library().moe_route(ctypes.byref(cfg), _ptr(x), T, ctypes.byref(weights), _ptr(logits),
                                    _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(ws), ws_bytes, _stream(stream))


def moe_forward(cfg, x, T, weights, y, y_dtype, aux, ws, ws_bytes, stream=None) -> int:
    return load_library().moe_forward(ctypes.byref(cfg), _ptr(x), T, ctypes.byref(weights), _ptr(y), y_dtype,
                                      None if aux is None else ctypes.byref(aux), _ptr(ws), ws_bytes,
                                      _stream(stream))


def moe_forward_timed(cfg, x, T, weights, y, y_dtype, aux, ws, ws_bytes, stream, stage_events) -> int:
    """stage_events: MOE_N_STAGES + 1 torch.cuda.Event(enable_timing=True)
    objects or None (that boundary is not recorded).

    torch creates an event's CUDA handle on its first record; events never
    recorded are recorded once here so that a valid handle is passed."""
    for e in stage_events:
        if e is not None and not e.cuda_event:
            e.record(torch.cuda.current_stream())
    arr = (ctypes.c_void_p * len(stage_events))(*[None if e is None else e.cuda_event for e in stage_events])
    return load_library().moe_forward_timed(ctypes.byref(cfg), _ptr(x), T, ctypes.byref(weights), _ptr(y), y_dtype,
                                            None if aux is None else ctypes.byref(aux), _ptr(ws), ws_bytes,
                                            _stream(stream), arr)


def moe_aux_stats(cfg, T, logits, topk_idx, topk_w, out, ws, ws_bytes, stream=None) -> int:
    return load_library().moe_aux_stats(ctypes.byref(cfg), T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                                        ctypes.byref(out), _ptr(ws), ws_bytes, _stream(stream))


def moe_aux_stats_noalloc(cfg, T, logits, topk_idx, topk_w, out, stream=None) -> int:
    """moe_aux_stats with its scratch in the library's fixed array instead of a
    workspace; for callers that cannot allocate.  Calls that overlap on the
    device race on that array."""
    return load_library().moe_aux_stats_noalloc(ctypes.byref(cfg), T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                                                ctypes.byref(out), _stream(stream))


def aux_partials_len(N: int) -> int:
    return 3 * N + 1


def moe_aux_partials(cfg, T, logits, topk_idx, topk_w, partials, stream=None) -> int:
    """One rank's statistics as exact int64 partial sums (device tensor of 3N+1)."""
    return load_library().moe_aux_partials(ctypes.byref(cfg), T, _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                                           _ptr(partials), _stream(stream))


def moe_aux_finalize(cfg, partials, out, stream=None) -> int:
    return load_library().moe_aux_finalize(ctypes.byref(cfg), _ptr(partials), ctypes.byref(out), _stream(stream))


def moe_aux_finalize_host(cfg, partials, counts=None, importance=None, p_mean=None, scalars=None) -> int:
    """Host version: partials, counts, importance, p_mean, scalars are CPU tensors (int64, int32, fp32)."""
    return load_library().moe_aux_finalize_host(ctypes.byref(cfg), _ptr(partials), _ptr(counts), _ptr(importance),
                                                _ptr(p_mean), _ptr(scalars))


def moe_ep_workspace_size(cfg, n_ranks, T) -> int:
    return load_library().moe_ep_workspace_size(ctypes.byref(cfg), n_ranks, T)


def moe_ep_dispatch(cfg, n_ranks, x, T, weights, send_x, send_expert, send_w, send_counts, send_pos, aux, ws,
                    ws_bytes, stream=None) -> int:
    return load_library().moe_ep_dispatch(ctypes.byref(cfg), n_ranks, _ptr(x), T, ctypes.byref(weights), _ptr(send_x),
                                          _ptr(send_expert), _ptr(send_w), _ptr(send_counts), _ptr(send_pos),
                                          None if aux is None else ctypes.byref(aux), _ptr(ws), ws_bytes,
                                          _stream(stream))


def moe_ep_experts_workspace_size(cfg_local, M) -> int:
    return load_library().moe_ep_experts_workspace_size(ctypes.byref(cfg_local), M)


def moe_ep_experts(cfg_local, recv_x, M, recv_expert, recv_w, weights_local, z_out, ws, ws_bytes, stream=None) -> int:
    return load_library().moe_ep_experts(ctypes.byref(cfg_local), _ptr(recv_x), M, _ptr(recv_expert), _ptr(recv_w),
                                         ctypes.byref(weights_local), _ptr(z_out), _ptr(ws), ws_bytes,
                                         _stream(stream))


def moe_ep_combine(cfg, z_back, T, send_pos, y, y_dtype, stream=None) -> int:
    return load_library().moe_ep_combine(ctypes.byref(cfg), _ptr(z_back), T, _ptr(send_pos), _ptr(y), y_dtype,
                                         _stream(stream))


def make_grads(dx, dW_g, dW1, dW2, db_g=None, db1=None, db2=None) -> moe_grads:
    return moe_grads(_ptr(dx), _ptr(dW_g), _ptr(db_g), _ptr(dW1), _ptr(db1), _ptr(dW2), _ptr(db2))


def moe_backward_workspace_size(cfg, T) -> int:
    return load_library().moe_backward_workspace_size(ctypes.byref(cfg), T)


def moe_backward(cfg, x, T, weights, dy, alpha_switch, alpha_importance, grads, ws, ws_bytes, stream=None) -> int:
    return load_library().moe_backward(ctypes.byref(cfg), _ptr(x), T, ctypes.byref(weights), _ptr(dy),
                                       float(alpha_switch), float(alpha_importance), ctypes.byref(grads), _ptr(ws),
                                       ws_bytes, _stream(stream))


def moe_get_workspace_layout(cfg, T) -> moe_workspace_layout:
    out = moe_workspace_layout()
    check(load_library().moe_get_workspace_layout(ctypes.byref(cfg), T, ctypes.byref(out)), "layout")
    return out


def moe_total_params(cfg) -> int:
    return load_library().moe_total_params(ctypes.byref(cfg))


def moe_active_params(cfg) -> int:
    return load_library().moe_active_params(ctypes.byref(cfg))


def moe_get_device_status() -> int:
    return load_library().moe_get_device_status()


def moe_launch_count() -> int:
    return load_library().moe_launch_count()


def moe_error_string(code: int) -> str:
    return error_string(code)


def moe_selftest_wait_timeout(timeout_ns: int, stream=None) -> int:
    return load_library().moe_selftest_wait_timeout(timeout_ns, _stream(stream))


def alloc_workspace(cfg: moe_config, T: int, device="cuda") -> torch.Tensor:
    """A device byte buffer of moe_workspace_size bytes (torch's allocator aligns blocks to 512 bytes)."""
    n = moe_workspace_size(cfg, T)
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)
