"""The multi-process path of bench.py on CPU: two gloo ranks (the layout
torchrun gives one process per GPU).  The path shards whole batches across
ranks with no collective on the data path, so what is tested is the plumbing:
every rank draws its own inputs, the step time is the max over ranks, and the
reported throughput adds all ranks' tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_, r_, l_ = bench.dist_env()
        assert (w_, r_, l_) == (world, rank, rank)
        # each rank times a different amount; the job time is the slowest one
        local_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(local_ms, world)
        # each rank draws its own batch of the same workload
        w = wl.shrink(wl.GRAFT_LAYER, n_heads=2, lengths=(128,))
        inp = wl.make_prefill_inputs(wl.shrink(w, seed=bench.rank_seed(w.seed, 0, rank)))
        digest = float(inp["q"].float().sum())
        t = torch.tensor([digest], dtype=torch.float64)
        allv = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allv, t)
        bench.barrier(world)
        out[rank] = (ms, [float(x) for x in allv],
                     bench.job_throughput(128, world, 10, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        ps = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0                       # max over ranks
    assert res[0][1][0] != res[0][1][1]                         # different batches
    assert res[0][2] == pytest.approx(2 * 128 * 10 / 15e-3)     # all ranks' tokens
