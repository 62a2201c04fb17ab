"""Host side of context-parallel decode on CPU: the exchange used between
ranks (torch.distributed all-gather, here over two gloo processes) stacks the
ranks' partials in rank order for every buffer shape and type the step
exchanges, and the position ranges of the shards."""
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_full_b200.context_parallel import nccl_all_gather, shard_offsets


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        gather = nccl_all_gather()
        B, Hq, D, rows, kk = 2, 4, 128, 2, 1152
        O_part = torch.full((B, Hq, D), float(rank) + 0.5)
        ml_part = torch.full((B, Hq, 2), -float(rank))
        pair_pos = torch.arange(rows * kk, dtype=torch.int32).view(rows, kk) + 100000 * rank
        got = [gather(O_part), gather(ml_part), gather(pair_pos)]
        q.put((rank, [g.numpy() for g in got]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_all_gather_stacks_partials_in_rank_order():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, got = q.get(timeout=120)
        res[r] = got
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        O, ml, pp = res[r]
        assert O.shape == (2, 2, 4, 128) and ml.shape == (2, 2, 4, 2) and pp.shape == (2, 2, 1152)
        for src in range(world):
            assert (O[src] == src + 0.5).all() and (ml[src] == -src).all()
            assert pp[src, 0, 0] == 100000 * src and pp.dtype == np.int32
    assert all(np.array_equal(a, b) for a, b in zip(res[0], res[1]))


def test_shard_offsets():
    lens = [[2000, 1200], [1500, 1240], [2500, 60]]
    pos0 = shard_offsets(lens)
    assert pos0.tolist() == [[0, 0], [2000, 1200], [3500, 2440]]
    # the ranges of a sequence tile it in rank order
    n = np.asarray(lens)
    assert ((pos0 + n)[:-1] == pos0[1:]).all()
    assert ((pos0 + n)[-1] == n.sum(axis=0)).all()
