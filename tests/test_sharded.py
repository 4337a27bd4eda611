"""Host side of the vocabulary-sharded heads: the row split and the exchange
of the partials (all-gather in rank order), with two gloo ranks on CPU."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from medusa_tree_speculative_heads_b200.sharded import exchange_partials, vocab_shard


@pytest.mark.parametrize("V,world", [(128256, 8), (32000, 3), (1000, 7), (9, 9), (10, 4)])
def test_vocab_shards_tile_the_vocabulary_in_rank_order(V, world):
    shards = [vocab_shard(V, world, r) for r in range(world)]
    assert shards[0][0] == 0 and shards[-1][1] == V
    for (a0, a1), (b0, b1) in zip(shards, shards[1:]):
        assert a1 == b0                                   # contiguous, rank order
    sizes = [b - a for a, b in shards]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_vocab_shard_refuses_impossible_splits():
    for args in ((3, 4, 0), (10, 0, 0), (10, 2, 2), (10, 2, -1)):
        with pytest.raises(ValueError):
            vocab_shard(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    B, K = 3, 4
    # every byte names its rank and position
    local = ((torch.arange(B * K * 72) + 7 * rank) % 251).to(torch.uint8).reshape(B, K, 72)
    parts = exchange_partials(local)
    q.put((rank, parts.shape, [int(parts[r].to(torch.int64).sum()) for r in range(world)],
           all(torch.equal(parts[r], ((torch.arange(B * K * 72) + 7 * r) % 251).to(torch.uint8).reshape(B, K, 72))
               for r in range(world))))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_exchange_partials_in_rank_order():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shape, sums, ok in out:
        assert tuple(shape) == (2, 3, 4, 72) and ok
    assert out[0][2] == out[1][2]                        # both ranks hold the same gathered set
