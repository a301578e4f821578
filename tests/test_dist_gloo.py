"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, barriers,
the max-over-ranks timing reduction and the sharding of independent
sequences (no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_sparse_09_b200 import dist as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, nranks, port, out):
    os.environ.update(WORLD_SIZE=str(nranks), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    D.init("gloo", timeout_s=60)
    D.barrier()
    # each rank reports its own time; every rank must see the slowest
    mine = 1.0 + rank * 0.5
    out[rank] = (D.max_over_ranks(mine), list(D.shard(10, rank, nranks)), D.seed_offset(rank))
    D.barrier()
    D.finalize()


@pytest.mark.parametrize("nranks", [2])
def test_gloo_two_ranks(nranks):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, nranks, port, out)) for r in range(nranks)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 1.5
    shards = [out[r][1] for r in range(nranks)]
    assert sorted(sum(shards, [])) == list(range(10))
    assert out[0][2] != out[1][2]


def test_single_rank_is_identity():
    assert D.max_over_ranks(3.0) == 3.0
    assert list(D.shard(7, 0, 1)) == list(range(7))
