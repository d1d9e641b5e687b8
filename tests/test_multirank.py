"""The N > 1 path on the CPU: world-size-2 gloo ranks each take their shard
(block-aligned ranges from dequantization_bq_quantize_b200.shard), compute it
with the oracle, and the gathered shards must equal the single-process result;
the max-over-ranks timing reduction is checked the same way."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dequantization_bq_quantize_b200 import shard


def test_block_ranges_cover_and_align():
    for n in (0, 1, 63, 64, 65, 1000, 8388645):
        for bs in (32, 64, 4096):
            for world in (1, 2, 3, 8):
                rs = shard.block_ranges(n, bs, world)
                assert len(rs) == world
                assert rs[0][0] == 0 and rs[-1][1] == n
                for (a, b), (c, _) in zip(rs, rs[1:]):
                    assert b == c
                for lo, hi in rs:
                    assert lo % bs == 0 and lo <= hi
                    assert hi == n or hi % bs == 0


def test_shard_offsets():
    assert shard.shard_offsets(128, 200, 64, 16) == (2, 2, 64, 36)
    assert shard.shard_offsets(128, 200, 64, 256) == (2, 2, 128, 72)
    with pytest.raises(ValueError):
        shard.shard_offsets(100, 200, 64, 16)


def test_gguf_ranges():
    rs = shard.gguf_ranges(1835008, 8)
    assert rs[0][0] == 0 and rs[-1][1] == 1835008
    assert sum(b - a for a, b in rs) == 1835008


def _worker(rank, world, port, n, bs, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from bq_inputs import codebooks, synth
        x = synth.to_numpy_bits(synth.sweep("bf16", bs, seed=7, n=n))
        table = codebooks.nf4()
        lo, hi = shard.block_ranges(n, bs, world)[rank]
        a, q = oracle.quantize_blockwise(x[lo:hi], "bf16", bs, table)
        # gather variable-length shards through padded tensors
        sizes = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([a.size, q.size]))
        ma = max(int(s_[0]) for s_ in sizes)
        mq = max(int(s_[1]) for s_ in sizes)
        ta = torch.zeros(ma, dtype=torch.float32)
        ta[:a.size] = torch.from_numpy(a)
        tq = torch.zeros(mq, dtype=torch.uint8)
        tq[:q.size] = torch.from_numpy(q)
        ga = [torch.zeros(ma, dtype=torch.float32) for _ in range(world)]
        gq = [torch.zeros(mq, dtype=torch.uint8) for _ in range(world)]
        dist.all_gather(ga, ta)
        dist.all_gather(gq, tq)
        # timing: the job's time is the slowest rank's
        t = torch.tensor([10.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            absmax = np.concatenate([g[:int(s_[0])].numpy() for g, s_ in zip(ga, sizes)])
            codes = np.concatenate([g[:int(s_[1])].numpy() for g, s_ in zip(gq, sizes)])
            ra, rq = oracle.quantize_blockwise(x, "bf16", bs, table)
            result["ok"] = bool(np.array_equal(absmax, ra) and np.array_equal(codes, rq))
            result["max_ms"] = float(t.item())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,bs", [(8192 * 3 + 37, 64), (4096 * 5 + 1, 4096)])
def test_two_rank_shards_equal_single_rank(n, bs):
    world = 2
    port = 29500 + (os.getpid() % 2000)
    with mp.Manager() as mgr:
        result = mgr.dict()
        mp.spawn(_worker, args=(world, port, n, bs, result), nprocs=world, join=True)
        assert result["ok"]
        assert result["max_ms"] == 11.0
        assert shard.aggregate_gbs(1e9, world, result["max_ms"]) == pytest.approx(2e9 / 11e-3 / 1e9)
