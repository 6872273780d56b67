"""Run a fixed set of layer calls through whichever build of the library the
environment selects (MOE_BOUNDS_CHECK=1: the bounds-check build) and save
their outputs and device status words, for test_gpu_bounds_check.py.

    python -m tests.bounds_child OUT_FILE
"""
import sys

import torch

import sparse_mixture_experts_10_b200 as moe
from moe_inputs import WORKLOADS, make_inputs

# (name, workload, tokens): layers over every kernel family the forward uses
CASES = [
    ("tiny", WORKLOADS["tiny"], 300),
    ("tiny_capacity_drop", WORKLOADS["tiny"].with_(capacity_factor=1.0), 300),
    ("tiny_capacity_reroute", WORKLOADS["tiny"].with_(capacity_factor=1.0, overflow=1), 300),
    ("gpt2", WORKLOADS["gpt2"], 2000),
    ("mixtral", WORKLOADS["mixtral"], 300),
    ("deepseek_zipf_n32", WORKLOADS["deepseek_zipf"].with_(N=32), 1024),
    ("deepseek_shared_n32", WORKLOADS["deepseek_shared"].with_(N=32), 512),
    ("decode1", WORKLOADS["decode1"], 1),
    ("decode8", WORKLOADS["decode8"], 8),
]


def layer_case(wl, T):
    inp = make_inputs(wl, "cuda", T=T)
    cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias, wl.n_shared,
                          wl.capacity_factor, wl.overflow)
    w = moe.make_weights(inp["W_g"], inp["W1"], inp["W2"], inp["b_g"], inp["b1"], inp["b2"], inp.get("b_sel"),
                         inp.get("S1"), inp.get("sb1"), inp.get("S2"), inp.get("sb2"))
    ws = moe.alloc_workspace(cfg, T)
    y = torch.empty(T, wl.D, device="cuda")
    moe.check(moe.moe_forward(cfg, inp["x"], T, w, y, moe.MOE_F32, None, ws, ws.numel()), "moe_forward")
    st = moe.moe_get_device_status()
    return y.cpu(), st


def combine_with_bad_row():
    """moe_ep_combine with one send_pos entry past z_back's T*K rows.  z_back is
    the head of a larger buffer, so that the row read in a build without the
    check is still inside an allocation (its rows hold 1e6)."""
    T, K, D = 64, 2, 256
    cfg = moe.make_config(D, 512, 8, K, moe.MOE_ACT_GELU, moe.MOE_F32)
    g = torch.Generator(device="cuda").manual_seed(5)
    zbig = torch.full(((T * K + 16), D), 1e6, device="cuda")
    zbig[:T * K] = torch.randn(T * K, D, generator=g, device="cuda")
    z_back = zbig[:T * K]
    pos = torch.randperm(T * K, generator=g, device="cuda").to(torch.int32)
    pos[3 * K + 1] = T * K + 5
    y = torch.empty(T, D, device="cuda")
    moe.check(moe.moe_ep_combine(cfg, z_back, T, pos, y, moe.MOE_F32), "moe_ep_combine")
    st = moe.moe_get_device_status()
    return y.cpu(), st


def main(out_file):
    moe.load_library()
    assert moe.moe_get_device_status() == 0
    res = {"lib": moe.LIB_PATH}
    for name, wl, T in CASES:
        res[name] = layer_case(wl, T)
        torch.cuda.empty_cache()
    if moe.LIB_PATH.endswith("libmoe_debug.so"):   # an invalid input goes to the checking build only
        res["combine_bad_row"] = combine_with_bad_row()
    torch.save(res, out_file)


if __name__ == "__main__":
    main(sys.argv[1])
