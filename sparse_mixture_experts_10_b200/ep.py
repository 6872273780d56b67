"""Expert parallelism: the exchange between the library's dispatch, expert and
combine calls (include/moe.h, moe_ep_*).

The experts are split over the ranks of a process group on dim 0.  Every rank
routes and packs its own tokens (moe_ep_dispatch), the packed rows travel to
the ranks holding their experts (an all-to-all over torch.distributed: NCCL
between GPUs, gloo between CPU processes), each rank evaluates its experts on
what it received (moe_ep_experts), the outputs travel back (the reverse
all-to-all) and each rank adds its tokens' rows in slot order
(moe_ep_combine).  This module only moves buffers and calls the C entry
points; every step of the layer runs in the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (check, moe_ep_combine, moe_ep_dispatch, moe_ep_experts, moe_ep_experts_workspace_size,
               moe_ep_workspace_size, MOE_F32)


def exchange(rows, send_counts, group=None):
    """All-to-all of rows grouped by destination rank (rank after rank, send_counts[r] rows
    for rank r).  Returns the received rows (source rank after source rank) and the counts
    received from each rank."""
    counts = send_counts.to(torch.int64)
    recv_counts = torch.empty_like(counts)
    dist.all_to_all_single(recv_counts, counts, group=group)
    ins, outs = counts.tolist(), recv_counts.tolist()
    recv = rows.new_empty((sum(outs),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(recv, rows[:sum(ins)].contiguous(), outs, ins, group=group)
    return recv, recv_counts


def exchange_back(rows, recv_counts, send_counts, group=None):
    """The reverse all-to-all: rows received from each rank go back to it, in the same order."""
    ins = recv_counts.to(torch.int64).tolist()
    outs = send_counts.to(torch.int64).tolist()
    back = rows.new_empty((sum(outs),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(back, rows.contiguous(), outs, ins, group=group)
    return back


def ep_forward(cfg, cfg_local, x, weights_router, weights_local, y, group=None, aux=None):
    """The layer under expert parallelism on this rank's tokens x [T, D]: dispatch, exchange,
    local experts, exchange back, combine into y [T, D] (fp32)."""
    R = dist.get_world_size(group)
    T, D, K = x.shape[0], cfg.DModel, cfg.TopK
    dev = x.device
    ws = torch.empty(max(moe_ep_workspace_size(cfg, R, T), 1), dtype=torch.uint8, device=dev)
    send_x = torch.empty(T * K, D, dtype=x.dtype, device=dev)
    send_e = torch.empty(T * K, dtype=torch.int32, device=dev)
    send_w = torch.empty(T * K, dtype=torch.float32, device=dev)
    send_counts = torch.empty(R, dtype=torch.int32, device=dev)
    send_pos = torch.empty(T * K, dtype=torch.int32, device=dev)
    check(moe_ep_dispatch(cfg, R, x, T, weights_router, send_x, send_e, send_w, send_counts, send_pos, aux, ws,
                          ws.numel()), "ep dispatch")
    recv_x, recv_counts = exchange(send_x, send_counts, group)
    recv_e, _ = exchange(send_e, send_counts, group)
    recv_w, _ = exchange(send_w, send_counts, group)
    M = recv_x.shape[0]
    z = torch.empty(M, D, dtype=torch.float32, device=dev)
    wsl = torch.empty(max(moe_ep_experts_workspace_size(cfg_local, M), 1), dtype=torch.uint8, device=dev)
    check(moe_ep_experts(cfg_local, recv_x, M, recv_e, recv_w, weights_local, z, wsl, wsl.numel()), "ep experts")
    z_back = exchange_back(z, recv_counts, send_counts, group)
    check(moe_ep_combine(cfg, z_back, T, send_pos, y, MOE_F32), "ep combine")
    return y
