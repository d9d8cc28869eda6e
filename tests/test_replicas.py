"""Replica sharding of the bench (N > 1 path) with world_size-2 gloo processes on CPU.

Each rank decodes its own shard of sequences with the fp64 oracle (standing in
for a GPU engine: the sharding logic is what is under test); the union must
equal the single-process result, and timing reduces to the maximum.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _decode(ids):
    from oracle.model import OracleModel
    from oracle.policies import OracleSequence
    from workload import CONFIGS, WeightSet, prefix_bytes

    wl = CONFIGS["tiny_d4"]
    m = OracleModel(wl.shape, WeightSet(wl.shape))
    out = []
    for i in ids:
        o = OracleSequence(m, wl, i, [int(b) for b in prefix_bytes(wl.seed, wl.cfg_index, i, wl.prefix_len)])
        o.prefill()
        out.append((i, o.generate(8)))
    return out


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    from block_diffusion_byte_b200.replicas import gather_lists, max_over_ranks, shard_ids

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = gather_lists(_decode(shard_ids(rank, world, 2)))
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            q.put((got, t))
    finally:
        dist.destroy_process_group()


def test_shard_ids():
    from block_diffusion_byte_b200.replicas import shard_ids

    assert shard_ids(0, 2, 3) == [0, 1, 2] and shard_ids(1, 2, 3) == [3, 4, 5]
    with pytest.raises(ValueError):
        shard_ids(2, 2, 1)


def test_two_gloo_ranks_equal_one_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got, t = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert t == 2.0  # max over ranks
    assert got == _decode([0, 1, 2, 3])
