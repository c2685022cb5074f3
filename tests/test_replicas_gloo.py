"""Multi-GPU runs are independent replicas (the decode step has no cross-GPU exchange):
each rank runs its own workload and the job's throughput is all ranks' tokens over the
slowest rank's time. This checks that host-side logic with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import bench
    import workloads as WL
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank timings differ; the reduction must return the max on every rank
        mine = [10.0 + rank, 5.0 - rank, 1.0 * rank]
        got = bench.reduce_max_over_ranks(mine, True)
        # replicas use different seeds: their workloads differ but have the same shapes
        cfg = WL.small_config(B=2)
        lay = WL.block_layout(cfg, seed=rank)
        q.put((rank, got, bench.replica_throughput(cfg.B, world, got[0] / 10), lay.seq_lens))
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, g0, v0, l0), (r1, g1, v1, l1) = res
    assert g0 == g1 == [11.0, 5.0, 1.0]
    # 2 sequences per rank x 2 ranks over the slowest rank's 1.1 ms per step
    assert abs(v0 - 2 * 2 / 1.1e-3) < 1e-6 and v0 == v1
    assert l0 != l1
