"""Multi-process (gloo, world size 2) checks of the row-sharded path's host logic.

Each rank draws its rows from the row-keyed generator; together the shards must
reproduce, bit for bit and in order, the batch a single process draws, and the
timing reduction must return the maximum over ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from invariant_bi_matmul_02_b200 import inputs
from invariant_bi_matmul_02_b200.shard import max_over_ranks, shard_rows, weak_rows


def test_shard_rows_partition():
    for total in (0, 1, 7, 1024, 1025):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    assert weak_rows(1024, 3) == (3072, 4096)
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, total, cols, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        start, stop = shard_rows(total, world, rank)
        mine = inputs.rows_normal(77, start, stop - start, cols)
        gathered = [None] * world
        dist.all_gather_object(gathered, (start, stop, inputs.bf16_bits(mine).tobytes()))
        t = max_over_ranks(10.0 + rank)
        if rank == 0:
            torch.save({"gathered": gathered, "max": t}, result_path)
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reproduce_single_process_batch(tmp_path):
    world, total, cols = 2, 37, 64
    out = str(tmp_path / "res.pt")
    mp.start_processes(_worker, args=(world, _free_port(), total, cols, out), nprocs=world,
                       join=True, start_method="spawn")
    res = torch.load(out)
    assert res["max"] == 11.0
    whole = inputs.bf16_bits(inputs.rows_normal(77, 0, total, cols)).tobytes()
    parts = sorted(res["gathered"])
    assert parts[0][0] == 0 and parts[-1][1] == total
    assert b"".join(p[2] for p in parts) == whole
