"""Host logic of the vocabulary sharding: the split, and the two exchanges
(all-gather of per-shard results, max all-reduce of candidate logits) run by
two gloo ranks on the CPU."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_medusa_b200 import sharded as S


@pytest.mark.parametrize("V,world", [(128256, 8), (32000, 3), (10, 4), (7, 7), (5, 2)])
def test_shard_range_partitions_the_vocabulary(V, world):
    ranges = [S.shard_range(V, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == V
    for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1
    assert S.shard_offsets(V, world) == [a for a, _ in ranges]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rec = torch.full((6, 4), float(rank))
        rec[:, 1] = 100 + rank
        stacked = S.gather_stacked(rec)
        cand = torch.tensor([float("-inf"), rank * 1.0, 5.0 - rank, float("-inf")])
        S.max_over_ranks(cand)
        out[rank] = (stacked.tolist(), cand.tolist())
    finally:
        dist.destroy_process_group()


def test_exchanges_with_two_gloo_ranks():
    world = 2
    port = 29500 + os.getpid() % 1000
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    for rank in range(world):
        stacked, cand = res[rank]
        assert len(stacked) == world
        for g in range(world):
            assert all(row[0] == float(g) and row[1] == 100 + g for row in stacked[g])
        assert cand == [float("-inf"), 1.0, 5.0, float("-inf")]
