"""Layer sharding of the warmup: host logic on CPU with gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_absorption_b200.sharding import gather_errors, owned_layers


def test_owned_layers_partition_all_layers():
    for L in (1, 5, 30, 40):
        for world in (1, 2, 3, 8):
            parts = [owned_layers(L, world, r) for r in range(world)]
            flat = sorted(l for p in parts for l in p)
            assert flat == list(range(L))
            assert all(p == sorted(p) for p in parts)
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    with pytest.raises(ValueError):
        owned_layers(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, L, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = owned_layers(L, world, rank)
        # each rank "computes" the errors of its layers: layer l -> (l, 1/(l+1))
        err = torch.tensor([[float(l), 1.0 / (l + 1)] for l in mine], dtype=torch.float64)
        full = gather_errors(err.reshape(-1, 2), L, world)
        q.put((rank, full.numpy().tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L", [(2, 5), (2, 30), (3, 7)])
def test_gather_errors_gives_every_rank_the_full_table(world, L):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [[float(l), 1.0 / (l + 1)] for l in range(L)]
    for rank, table in got:
        assert np.array_equal(np.array(table), np.array(want)), rank
