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


def _decode_oracle(wl, inp, seqs):
    """Index, top-k and attention of the oracle for the given sequences of a
    decode batch: {b: (selected indices, output)}."""
    import numpy as np
    from oracle import pipeline as P
    res = {}
    sink = inp["sink"].double().numpy()
    for b in seqs:
        pos = inp["q_pos"][b:b + 1].numpy()
        kv = P.cache_values(inp["ckv"][b], None, wl.kv, wl.c, wl.rope_dims)
        win = P.cache_values(inp["win"][b], None, wl.kv, wl.c, wl.rope_dims)
        idx, _, _, _ = P.select(wl, pos, inp["qI"][b:b + 1].double().numpy(),
                                inp["w"][b:b + 1].double().numpy(),
                                inp["kI"][b].double().numpy())
        out, _ = P.attend_wl(wl, pos, inp["q"][b:b + 1].double().numpy(), idx, kv, win,
                             int(inp["win_pos0"][b]), sink)
        res[b] = (np.asarray(idx), np.asarray(out))
    return res


def _shard_worker(rank, nranks, port, out):
    import torch.distributed as dist
    from long_context_sparse_09_b200 import synth
    from long_context_sparse_09_b200.configs import WORKLOADS
    os.environ.update(WORLD_SIZE=str(nranks), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    D.init("gloo", timeout_s=60)
    wl = WORKLOADS["tiny_csa_prefill_f32"]
    inp = synth.decode_inputs(wl, B=5)  # the same seeded batch on every rank
    mine = _decode_oracle(wl, inp, D.shard(5, rank, nranks))
    gathered = [None] * nranks
    dist.all_gather_object(gathered, mine)
    if rank == 0:
        merged = {}
        for part in gathered:
            assert not set(part) & set(merged)  # disjoint shares
            merged.update(part)
        out["merged"] = {b: (v[0].tolist(), v[1].tolist()) for b, v in merged.items()}
    D.barrier()
    D.finalize()


def test_two_ranks_decode_shares_match_one_process():
    """Two gloo ranks each take their share of a batch of decode sequences
    through the oracle's index, top-k and attention; the gathered results
    are those of one process over the whole batch."""
    import numpy as np
    from long_context_sparse_09_b200 import synth
    from long_context_sparse_09_b200.configs import WORKLOADS
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    merged = out["merged"]
    wl = WORKLOADS["tiny_csa_prefill_f32"]
    whole = _decode_oracle(wl, synth.decode_inputs(wl, B=5), range(5))
    assert sorted(merged) == list(range(5))
    for b in range(5):
        assert np.array_equal(np.asarray(merged[b][0]), whole[b][0])
        assert np.array_equal(np.asarray(merged[b][1]), whole[b][1])
