"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/moe.h declares, rejects bad arguments before touching
the device, and sizes its workspace consistently."""
import ctypes
import os
import re

import pytest

import oracle
import sparse_mixture_experts_10_b200 as moe
from sparse_mixture_experts_10_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def header_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_function_is_exported(lib):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(moe.EXPORTED) == names


def test_bounds_check_build_exports_the_same_functions():
    """The bounds-check build (-DMOE_DEBUG_BOUNDS, loaded under MOE_BOUNDS_CHECK=1) is the same
    library with index checks compiled in: it builds for sm_100a and exports every declared function."""
    path = moe_build.build(bounds_check=True)
    assert path.endswith("libmoe_debug.so") and path != moe_build.LIB
    dbg = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(dbg, n), n


def test_struct_sizes_match_header_layout():
    assert ctypes.sizeof(moe.moe_config) == 10 * 4
    assert ctypes.sizeof(moe.moe_weights) == 11 * 8
    assert ctypes.sizeof(moe.moe_aux) == 4 * 8
    assert ctypes.sizeof(moe.moe_workspace_layout) == 12 * 8 + 8 + 8


def cfg(D=64, H=256, N=8, K=2, act=moe.MOE_ACT_GELU, dtype=moe.MOE_F32, bias=True):
    return moe.make_config(D, H, N, K, act, dtype, bias)


@pytest.mark.parametrize("bad", [
    dict(D=0), dict(H=-1), dict(N=0), dict(K=0), dict(K=9), dict(N=2000, K=2), dict(N=64, K=33),
    dict(act=5), dict(dtype=7), dict(D=66, dtype=moe.MOE_F32), dict(D=100, dtype=moe.MOE_BF16),
    dict(H=12, dtype=moe.MOE_BF16),
])
def test_invalid_config_rejected(lib, bad):
    c = cfg(**bad)
    assert moe.moe_workspace_size(c, 16) == 0
    rc = moe.moe_forward(c, 16, 16, moe.make_weights(16, 16, 16), 16, moe.MOE_F32, None, 256, 1 << 30, 0)
    assert rc in (moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_UNSUPPORTED)


def test_overflow_policy_values(lib):
    """overflow takes the two documented values only; with a capacity either sizes the workspace."""
    for ov in (moe.MOE_OVERFLOW_DROP, moe.MOE_OVERFLOW_REROUTE):
        c = moe.make_config(64, 256, 8, 2, moe.MOE_ACT_GELU, moe.MOE_BF16, False, capacity_factor=1.0, overflow=ov)
        assert moe.moe_workspace_size(c, 4096) > 0
    for ov in (-1, 2, 7):
        c = moe.make_config(64, 256, 8, 2, moe.MOE_ACT_GELU, moe.MOE_BF16, False, capacity_factor=1.0, overflow=ov)
        assert moe.moe_workspace_size(c, 4096) == 0


def test_swiglu_with_bias_is_unsupported(lib):
    c = cfg(act=moe.MOE_ACT_SWIGLU, bias=True)
    assert moe.moe_forward(c, 16, 4, moe.make_weights(16, 16, 16), 16, 0, None, 256, 1 << 30, 0) == \
        moe.MOE_ERR_UNSUPPORTED


def test_argument_errors_before_any_launch(lib):
    c = cfg()
    W = moe.make_weights(256, 256, 256, b1=256, b2=256)
    need = moe.moe_workspace_size(c, 32)
    # null weights, null x, misaligned pointers, small workspace, negative T, bad y dtype
    assert moe.moe_forward(c, 256, 32, moe.make_weights(None, 256, 256), 256, 0, None, 256, need, 0) == \
        moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(c, None, 32, W, 256, 0, None, 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(c, 258, 32, W, 256, 0, None, 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(c, 256, 32, W, 256, 0, None, 512 + 16, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(c, 256, 32, W, 256, 0, None, 256, need - 1, 0) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert moe.moe_forward(c, 256, -1, W, 256, 0, None, 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(c, 256, 32, W, 256, 9, None, 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    # biases declared but missing
    assert moe.moe_forward(c, 256, 32, moe.make_weights(256, 256, 256), 256, 0, None, 256, need, 0) == \
        moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route(c, 256, 32, W, None, None, 256, None, 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route(c, 256, 32, W, None, 256, 256, None, 256, need - 256, 0) == \
        moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert moe.moe_aux_stats(c, 32, None, 256, 256, moe.make_aux(), 256, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_selftest_wait_timeout(0, 0) == moe.MOE_ERR_INVALID_ARG


def test_zero_tokens_without_outputs_is_a_host_noop(lib):
    c = cfg()
    W = moe.make_weights(256, 256, 256, b1=256, b2=256)
    assert moe.moe_forward(c, None, 0, W, None, 0, None, None, 0, 0) == moe.MOE_OK


def test_workspace_layout_is_aligned_and_disjoint(lib):
    for c, T in [(cfg(), 512), (cfg(768, 3072, 6, 2, dtype=moe.MOE_BF16), 8192),
                 (cfg(7168, 2048, 256, 8, moe.MOE_ACT_SWIGLU, moe.MOE_BF16, False), 16384),
                 (cfg(2880, 2880, 32, 4, moe.MOE_ACT_SWIGLU, moe.MOE_BF16, False), 1)]:
        L = moe.moe_get_workspace_layout(c, T)
        assert L.total == moe.moe_workspace_size(c, T)
        assert L.row_align == 128
        assert L.rows_cap % 128 == 0 and L.rows_cap >= T * c.TopK + c.NExperts * 127
        offs = [L.logits, L.topk_idx, L.topk_w, L.counts, L.offsets, L.row_offsets, L.perm_slot, L.slot_row,
                L.x_perm, L.h, L.z]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs) and L.z < L.total
        es = 4 if c.dtype == moe.MOE_F32 else 2
        assert L.h - L.x_perm >= L.rows_cap * c.DModel * es
        assert L.z - L.h >= L.rows_cap * c.DHidden * es


@pytest.mark.parametrize("D,H,N,K,act,bias", [(64, 256, 8, 2, 0, 1), (768, 3072, 6, 2, 0, 1),
                                              (4096, 14336, 8, 2, 1, 0), (7168, 2048, 256, 8, 1, 0)])
def test_param_accounting_agrees_with_oracle(lib, D, H, N, K, act, bias):
    c = cfg(D, H, N, K, act, moe.MOE_BF16, bias)
    assert moe.moe_total_params(c) == oracle.total_params(D, H, N, K, act, bias)
    assert moe.moe_active_params(c) == oracle.active_params(D, H, N, K, act, bias)


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -99):
        assert isinstance(moe.moe_error_string(code), str) and moe.moe_error_string(code)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        moe.load_library()
