"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode path shards by sequence with no data-path collective: each rank
owns its own batch, and the only cross-rank steps are the barrier and the
max-over-ranks reduction of the timed duration.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import sikv_inputs as gen

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        w = bench.shard_workload(gen.small(1, n=300, batch=2, num_q_heads=8, num_kv_heads=2), rank)
        hi = gen.head_inputs(w, 0, 0)
        bench.barrier(world)
        t = bench.max_over_ranks(1.5 + rank, world)
        results[rank] = (t, w.seed, hi.keys[:4].copy(), w.batch)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_take_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 2.5                      # max over ranks
    assert r0[1] != r1[1]                             # each rank decodes its own sequences
    assert not np.array_equal(r0[2], r1[2])
    assert r0[3] == r1[3]                             # same per-rank work (weak scaling)


def test_step_bytes_formula():
    import bench
    import sikv_inputs as gen

    w = gen.config(2)
    per = 16 * (131072 - 64) + 2048 * 128 * 2 + 64 * 2 * 128 * 2 + 8192
    assert bench.step_bytes(w) == per * 32 == 85_164_032
