"""The multi-rank path of bench.py on CPU ranks (gloo, world size 2): each rank
draws its own batch, the job time is the maximum over ranks, and the
throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from moe_inputs import WORKLOADS, make_inputs

        wl = WORKLOADS["tiny"]
        seed = bench.rank_seed(wl, rank)
        x = make_inputs(wl, "cpu", T=16, seed=seed)["x"]
        gathered = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        my_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(my_ms, torch.device("cpu"), world)
        tps = bench.job_throughput(wl.T, world, 7, mx)
        q.put((rank, seed, not torch.equal(gathered[0], gathered[1]), mx, tps))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_shard_and_take_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, diff0, mx0, t0), (r1, s1, diff1, mx1, t1) = res
    assert s0 != s1 and diff0 and diff1          # distinct batches per rank
    assert mx0 == mx1 == 15.0                    # slowest rank's time on every rank
    assert t0 == t1 == pytest.approx(512 * 2 * 7 / 0.015)
