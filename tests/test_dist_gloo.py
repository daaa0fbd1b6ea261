"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2):
the path shards as independent layers per rank (weak scaling, no data-path
collective); the only collectives are the timing barrier and the max over
ranks of the device time."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        w = synth.make_prefill("tiny-1h-1k-d64", device="cpu", seed=bench.rank_seed("tiny-1h-1k-d64", rank))
        digest = float(w.q.float().sum())
        t = torch.tensor([digest], dtype=torch.float64)
        all_d = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_d, t)
        out[rank] = (got, [float(x) for x in all_d])
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_independent_shards():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 15.0          # max over ranks
    d0, d1 = out[0][1]
    assert d0 != d1                                # each rank owns a different layer
