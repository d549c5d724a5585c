"""Multi-process host logic on CPU (gloo, world size 2): shard assignment and
max-over-ranks timing, the two pieces a multi-GPU bench run relies on."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_154_b200 import dist as fdist
from exact_attention_154_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = fdist.shard_workload(synth.single_head_n256(), world, rank)
        t = fdist.max_over_ranks(10.0 + rank, world)
        fdist.barrier(world)
        seeds = [None] * world
        dist.all_gather_object(seeds, w.seed)
        q.put((rank, t, seeds, w.B, w.N))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, seeds, B, N in results:
        assert t == 11.0                       # max over ranks
        assert len(set(seeds)) == world        # distinct shards
        assert (B, N) == (1, 256)              # per-GPU shape unchanged (weak scaling)


def test_shard_single_rank_is_identity():
    w = synth.seqlen_sweep(4096, False)
    assert fdist.shard_workload(w, 1, 0) == w
    with pytest.raises(ValueError):
        fdist.shard_workload(w, 2, 2)
