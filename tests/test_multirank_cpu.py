"""The N > 1 bench path on CPU: world_size-2 gloo ranks run the timing
aggregation the bench uses (barrier, max over ranks) and the token-shard
seeding (each rank draws its own activations)."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import synth
    ms = 10.0 + 5.0 * rank                       # each rank's own elapsed time
    agg = bench.max_over_ranks(ms, world, torch.device("cpu"))
    x = synth.normal_bf16_bits((4, 64), rank, synth.STREAM_X)
    q.put((rank, agg, x.tobytes()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_and_shards():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert all(agg == 15.0 for _, agg, _ in res)          # the max over ranks
    assert res[0][2] != res[1][2]                          # distinct token shards
    assert bench.tokens_per_s(2048, 20, 15.0, world) == 2 * 2048 * 20 / 0.015


import bench  # noqa: E402  (module-level import after the spawn helpers)
