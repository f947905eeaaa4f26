"""Host-side multi-rank logic on CPU (gloo, world size 2): no GPU needed."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from linear_attention_rnn_wkv7_b200 import replicas


def test_partition_sequences_balances_tokens():
    lengths = [8192, 16, 4000, 4100, 50, 7000, 900, 1]
    parts = replicas.partition_sequences(lengths, 2)
    assert sorted(i for p in parts for i in p) == list(range(len(lengths)))
    loads = [sum(lengths[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(lengths)
    assert replicas.partition_sequences([], 3) == [[], [], []]
    assert replicas.partition_sequences([5, 5], 1) == [[0, 1]]


def test_replica_seed():
    assert replicas.replica_seed(7, 0) == 7
    assert len({replicas.replica_seed(7, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = replicas.max_over_ranks(1.5 + rank)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_max_over_ranks_without_group():
    assert replicas.max_over_ranks(3.25) == 3.25
