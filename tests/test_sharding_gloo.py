"""Multi-rank path on CPU: two gloo ranks each run the mixer (here the CPU
oracle, standing in for one GPU per rank) on their share of a packed batch;
gathering the shares reproduces the unsharded result exactly. No collective
is on the data path -- only the final gather used by this check."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_linear_silu_b200.sharding import assign_sequences, shard_tokens


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(Hk=2):
    import gdn_inputs as gi
    return gi.random_prefill(41, [50, 3, 0, 120, 77, 9, 64], H=2, Hk=Hk, dk=8, dv=8, dtype="f32",
                             with_h0=True)


def _rank_main(rank, world, port, q, Hk=2):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        P = _problem(Hk)
        lens = np.diff(P.cu_seqlens)
        mine = assign_sequences(lens, world)[rank]
        tok, cu = shard_tokens(P.cu_seqlens, mine)
        o, hT = oracle.recurrence(P.q[tok], P.k[tok], P.v[tok], P.g[tok], P.beta[tok], cu,
                                  dtype=P.dtype, h0=P.h0[mine], threads=1)
        payload = [None] * world
        dist.all_gather_object(payload, (mine, tok, o, hT))
        if rank == 0:
            q.put(payload)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Hk", [2, 1], ids=["plain", "grouped_heads"])
def test_sequence_sharding_matches_unsharded(Hk):
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, Hk)) for r in range(world)]
    for p in procs:
        p.start()
    payload = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    P = _problem(Hk)
    o_ref, h_ref = oracle.recurrence(P.q, P.k, P.v, P.g, P.beta, P.cu_seqlens, dtype=P.dtype,
                                     h0=P.h0, threads=1)
    o = np.full_like(o_ref, np.nan)
    hT = np.full_like(h_ref, np.nan)
    seen = []
    for mine, tok, o_r, h_r in payload:
        o[tok] = o_r
        hT[mine] = h_r
        seen += mine
    assert sorted(seen) == list(range(P.N))          # every sequence on exactly one rank
    assert np.array_equal(o, o_ref) and np.array_equal(hT, h_ref)


def test_assignment_is_balanced_and_complete():
    lens = [300, 10, 290, 5, 150, 150, 0]
    parts = assign_sequences(lens, 3)
    assert sorted(sum(parts, [])) == list(range(len(lens)))
    loads = [sum(lens[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(lens)
    with pytest.raises(ValueError):
        assign_sequences(lens, 0)
