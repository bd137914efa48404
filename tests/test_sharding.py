"""Head-parallel sharding over ranks (the multi-GPU path: no data exchange), checked
with world_size-2 gloo process groups on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_causal_attention_b200.sharding import shard_heads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, hq, hkv, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    h0, h1, g0, g1 = shard_heads(hq, hkv, rank, world)
    t = torch.tensor([h0, h1, g0, g1], dtype=torch.int64)
    out = [torch.zeros(4, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(out, t)
    if rank == 0:
        q.put([o.tolist() for o in out])
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_shards_partition_heads_and_groups(world):
    hq, hkv = 128, 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, hq, hkv, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    heads, groups = [], []
    G = hq // hkv
    for h0, h1, g0, g1 in got:
        heads += list(range(h0, h1))
        groups += list(range(g0, g1))
        assert h0 == g0 * G and h1 == g1 * G  # a rank's query heads are exactly its groups' heads
    assert sorted(heads) == list(range(hq)) and sorted(groups) == list(range(hkv))


def test_shard_heads_rejects_uneven_split():
    with pytest.raises(ValueError):
        shard_heads(128, 8, 0, 3)
    with pytest.raises(ValueError):
        shard_heads(128, 8, 2, 2)
