"""The multi-rank path on CPU ranks (gloo, world size 2): each rank draws its
own batch, the job time is the maximum over ranks, the throughput counts every
rank's tokens; and the layer's statistics of the global batch come from each
rank's exact integer partials, all-reduced and finalised by the library on
every rank."""
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


def _fixed(v):
    """round(v * 2^32) of fp32 values, as the library's partials define it."""
    import numpy as np
    return np.rint(np.asarray(v, dtype=np.float32).astype(np.float64) * 4294967296.0).astype(np.int64)


def _stats_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np

        import oracle
        import sparse_mixture_experts_10_b200 as moe
        from moe_inputs import WORKLOADS, bf16_bits, make_inputs

        wl = WORKLOADS["tiny"].with_(zipf_s=0.7)
        T = 96 + 40 * rank                      # ragged shards
        inp = make_inputs(wl, "cpu", T=T, seed=100 + rank)
        inp["W_g"] = make_inputs(wl, "cpu", T=1, seed=7)["W_g"]   # weights replicated on every rank
        xr = oracle.load_rows(bf16_bits(inp["x"]), oracle.F32, range(T))
        sc = oracle.router_scores(xr, bf16_bits(inp["W_g"]), oracle.F32, bf16_bits(inp["b_g"]))
        lg = sc.astype(np.float32)              # the scores as a rank's device would hold them
        sel = oracle.select_topk(lg.astype(np.float64), wl.K)
        w = oracle.gate_weights(lg.astype(np.float64), sel).astype(np.float32)
        N, K = wl.N, wl.K
        part = np.zeros(3 * N + 1, dtype=np.int64)
        np.add.at(part, sel.ravel(), 1)
        np.add.at(part, N + sel.ravel(), _fixed(w.ravel()))
        for t in range(T):
            part[2 * N:3 * N] += _fixed(oracle.softmax(lg[t].astype(np.float64)))
        part[3 * N] = T
        pt = torch.from_numpy(part)
        dist.all_reduce(pt)                      # the exchange step: int64 sums, exact in any order
        cfg = moe.make_config(wl.D, wl.H, N, K, wl.act, moe.MOE_F32, wl.has_bias)
        out = dict(counts=torch.empty(N, dtype=torch.int32), importance=torch.empty(N),
                   p_mean=torch.empty(N), scalars=torch.empty(4))
        moe.check(moe.moe_aux_finalize_host(cfg, pt, **out))
        # the union batch on every rank, for the oracle's statistics over it
        shards = [None] * world
        dist.all_gather_object(shards, (lg, sel, w))
        st = oracle.aux_stats(np.concatenate([a for a, _, _ in shards]).astype(np.float64),
                              np.concatenate([b for _, b, _ in shards]),
                              np.concatenate([c for _, _, c in shards]).astype(np.float64), N)
        q.put((rank, {k: v.numpy().copy() for k, v in out.items()}, st, int(pt[-1])))
    except Exception as exc:  # reported to the parent instead of leaving it waiting
        q.put((rank, repr(exc), None, -1))
        raise
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_global_statistics():
    import numpy as np
    from sparse_mixture_experts_10_b200 import build as moe_build
    moe_build.build()    # the ranks load the library (its host-side finalisation needs no GPU)
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_stats_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for r in res:
        assert isinstance(r[1], dict), f"rank {r[0]} failed: {r[1]}"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, out0, st, t0), (_, out1, _, t1) = res
    assert t0 == t1 == 96 + 136                  # the global token count
    for k in out0:                               # every rank finalised the same bits
        assert np.array_equal(out0[k], out1[k]), k
    np.testing.assert_array_equal(out0["counts"], st["counts"].astype(np.int32))
    np.testing.assert_allclose(out0["importance"], st["importance"], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(out0["p_mean"], st["p_mean"], rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(out0["scalars"], [st["switch"], st["simple"], st["cv2_importance"], st["cv2_load"]],
                               rtol=1e-5, atol=1e-7)


def _ep_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_mixture_experts_10_b200 import ep

        # rank r sends counts[r][d] rows to rank d; a row holds (source rank, destination, index)
        counts = [[3, 2, 0], [1, 4, 2], [0, 1, 5]][rank][:world]
        rows = torch.tensor([[rank, d, i] for d, c in enumerate(counts) for i in range(c)], dtype=torch.float32)
        recv, recv_counts = ep.exchange(rows, torch.tensor(counts, dtype=torch.int32))
        # what a rank's experts do to a row (any function of the row alone)
        out = recv * 10.0 + 1.0
        back = ep.exchange_back(out, recv_counts, torch.tensor(counts, dtype=torch.int32))
        q.put((rank, recv.tolist(), recv_counts.tolist(), back.tolist(), rows.tolist()))
    except Exception as exc:
        q.put((rank, repr(exc), None, None, None))
        raise
    finally:
        dist.destroy_process_group()


def test_expert_parallel_exchange_round_trip():
    """The expert-parallel all-to-alls on CPU ranks (gloo, world size 3): every rank receives the
    rows destined to it, source rank after source rank in the order they were packed, and the
    reverse exchange returns each processed row to its place on its source rank."""
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    all_counts = [[3, 2, 0], [1, 4, 2], [0, 1, 5]]
    for rank, recv, recv_counts, back, rows in res:
        assert isinstance(recv, list), recv
        expect = [[src, rank, i] for src in range(world) for i in range(all_counts[src][rank])]
        assert recv == expect
        assert recv_counts == [all_counts[src][rank] for src in range(world)]
        assert back == [[v * 10.0 + 1.0 for v in row] for row in rows]
