"""The benchmark's data-parallel plumbing on CPU: two gloo ranks draw disjoint
shards of one global batch (identical to drawing the batch at once), and the
timing reduction returns the slowest rank's time."""
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        batch, context = 2, 640
        w = synth.decode_128k(batch=batch, first_seq=bench.rank_first_sequence(rank, batch),
                              context=context)
        elapsed = 10.0 + rank  # rank 1 is slower
        m = bench.max_over_ranks(elapsed, world, "cpu")
        value = bench.job_throughput(batch, world, 5, m)
        q.put((rank, w.k.copy(), w.q.copy(), m, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_timing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, k, qq, m, value = q.get(timeout=120)
        res[r] = (k, qq, m, value)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    full = synth.decode_128k(batch=4, first_seq=0, context=640)
    assert np.array_equal(np.concatenate([res[0][0], res[1][0]]), full.k)
    assert np.array_equal(np.concatenate([res[0][1], res[1][1]]), full.q)
    assert res[0][2] == res[1][2] == 11.0  # max over ranks
    assert res[0][3] == res[1][3] == 2 * 2 * 5 / 0.011
