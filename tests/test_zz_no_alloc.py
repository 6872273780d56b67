"""moe_aux_stats_noalloc: the statistics entry point whose scratch is a fixed
array inside the library, checked against moe_aux_stats on the same routing
results.

The file name puts it last in collection order; it must also pass on its own
in a fresh process, where its first call is the one that looks up the array's
device address.
"""
import ctypes

import pytest
import torch

import sparse_mixture_experts_10_b200 as moe


def _routing(T, N, K, seed):
    """Seeded routing results on the device: logits, top-k indices (descending
    score) and gate weights renormalised over the selected experts."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    logits = torch.randn(T, N, generator=g, dtype=torch.float32)
    top = torch.topk(logits, K, dim=1)
    w = torch.softmax(top.values, dim=1)
    return (logits.cuda(), top.indices.to(torch.int32).cuda(), w.cuda())


def _aux_out(N):
    return dict(counts=torch.full((N,), -1, dtype=torch.int32, device="cuda"),
                importance=torch.full((N,), -1.0, device="cuda"),
                p_mean=torch.full((N,), -1.0, device="cuda"),
                scalars=torch.full((4,), -1.0, device="cuda"))


def _assert_same_stats(got, want):
    # the tolerance of the statistics comparisons between entry points
    assert torch.equal(got["counts"], want["counts"])
    for k in ("importance", "p_mean", "scalars"):
        torch.testing.assert_close(got[k], want[k], rtol=1e-5, atol=1e-6)


@pytest.mark.gpu
@pytest.mark.parametrize("T,N,K", [(500, 6, 2), (3001, 32, 4), (1, 32, 4), (2000, 256, 8), (777, 100, 3)])
def test_noalloc_stats_match_workspace_entry_point(T, N, K):
    cfg = moe.make_config(64, 256, N, K, moe.MOE_ACT_GELU, moe.MOE_F32, False)
    logits, idx, w = _routing(T, N, K, seed=T * 1000 + N)
    want = _aux_out(N)
    ws = moe.alloc_workspace(cfg, T)
    moe.check(moe.moe_aux_stats(cfg, T, logits, idx, w, moe.make_aux(**want), ws, ws.numel()), "moe_aux_stats")
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row share the array: the second must not see the first's state
        got = _aux_out(N)
        moe.check(moe.moe_aux_stats_noalloc(cfg, T, logits, idx, w, moe.make_aux(**got)), "moe_aux_stats_noalloc")
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        _assert_same_stats(got, want)


@pytest.mark.gpu
def test_noalloc_stats_on_a_side_stream_and_empty_batch():
    T, N, K = 1000, 16, 2
    cfg = moe.make_config(64, 256, N, K, moe.MOE_ACT_GELU, moe.MOE_F32, False)
    logits, idx, w = _routing(T, N, K, seed=7)
    want = _aux_out(N)
    ws = moe.alloc_workspace(cfg, T)
    moe.check(moe.moe_aux_stats(cfg, T, logits, idx, w, moe.make_aux(**want), ws, ws.numel()))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    got = _aux_out(N)
    with torch.cuda.stream(side):
        moe.check(moe.moe_aux_stats_noalloc(cfg, T, logits, idx, w, moe.make_aux(**got), side))
    torch.cuda.synchronize()
    _assert_same_stats(got, want)
    empty = _aux_out(N)
    moe.check(moe.moe_aux_stats_noalloc(cfg, 0, None, None, None, moe.make_aux(**empty)))
    torch.cuda.synchronize()
    assert int(empty["counts"].abs().sum()) == 0
    assert float(empty["importance"].abs().sum()) == 0.0


def test_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    """The size check runs on the host before any CUDA call, so it needs no GPU."""
    L = moe.load_library()
    cfg = moe.make_config(64, 256, 256, 8, moe.MOE_ACT_GELU, moe.MOE_F32, False)
    T = 1 << 20   # 16384 blocks x 256 experts x 4 bytes x 3 arrays = 48 MiB of partials
    fake = ctypes.c_void_p(256)   # never dereferenced: the call returns first
    aux = moe.moe_aux()
    rc = L.moe_aux_stats_noalloc(ctypes.byref(cfg), T, fake, fake, fake, ctypes.byref(aux), None)
    assert rc == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert moe.MOE_NOALLOC_SCRATCH_BYTES == 2 << 20
