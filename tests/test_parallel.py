"""The data-parallel host logic (w4a4_mixed_precision_b200/parallel.py) on CPU:
token shards, and the collectives the multi-GPU bench and callers use, run as
two gloo ranks (the same torch.distributed calls run on NCCL on GPUs)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from w4a4_mixed_precision_b200 import parallel


@pytest.mark.parametrize("M,world", [(0, 1), (1, 2), (7, 2), (8192, 8), (13, 4), (3, 8)])
def test_token_shards_cover_every_row_once(M, world):
    seen = []
    sizes = []
    for r in range(world):
        a, b = parallel.token_shard(M, world, r)
        assert 0 <= a <= b <= M
        seen.extend(range(a, b))
        sizes.append(b - a)
    assert seen == list(range(M))
    assert max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)


def test_token_shard_rejects_bad_arguments():
    for args in [(4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ValueError):
            parallel.token_shard(*args)


def test_single_process_is_the_identity():
    assert parallel.max_over_ranks(2.5) == 2.5
    assert parallel.sum_over_ranks(3.0) == 3.0
    y = torch.arange(12.0).reshape(3, 4)
    assert torch.equal(parallel.gather_rows(y, 3), y)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, M, N, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = parallel.token_shard(M, world, rank)
        # each rank "computes" its own rows: row i holds i * 10 + column
        y_local = (torch.arange(a, b, dtype=torch.float32)[:, None] * 10
                   + torch.arange(N, dtype=torch.float32)[None, :])
        t_max = parallel.max_over_ranks(1.0 + rank)          # per-rank "elapsed"
        units = parallel.sum_over_ranks(float(b - a))         # rows processed
        y = parallel.gather_rows(y_local, M)
        out[rank] = (t_max, units, y.tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M", [7, 64])
def test_two_gloo_ranks(M):
    world, N = 2, 5
    with mp.Manager() as manager:
        out = manager.dict()
        ctx = mp.get_context("spawn")
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, M, N, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        expect = [[i * 10.0 + j for j in range(N)] for i in range(M)]
        for r in range(world):
            t_max, units, y = out[r]
            assert t_max == 2.0          # the slowest rank
            assert units == float(M)     # every row counted once
            assert y == expect           # rows back in token order on every rank
