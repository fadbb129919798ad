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


def _layer_problem():
    """Layer input x [T, C] (q | k | v, Hk = 1, H = 2, d = 8), taps, conv windows, gates."""
    import gdn_inputs as gi
    lens = [50, 3, 0, 120, 77, 2, 64]
    C = 2 * 1 * 8 + 2 * 8
    x, w, cu, st = gi.random_mixed(43, lens, C, K=4, dtype="f32", with_state=True)
    P = gi.random_prefill(43, lens, H=2, Hk=1, dk=8, dv=8, dtype="f32", with_h0=True)
    return x, w, cu, st, P


def _layer_oracle(x, w, cu, st, g, beta, h0):
    import oracle
    y, st_out = oracle.conv_silu(x, w, cu, dtype="f32", state_in=st, threads=1)
    T = y.shape[0]
    o, hT = oracle.recurrence(y[:, :8].reshape(T, 1, 8), y[:, 8:16].reshape(T, 1, 8),
                              y[:, 16:].reshape(T, 2, 8), g, beta, cu, dtype="f64", h0=h0, threads=1)
    return o, hT, st_out


def _layer_rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, w, cu, st, P = _layer_problem()
        mine = assign_sequences(np.diff(cu), world)[rank]
        tok, cu_r = shard_tokens(cu, mine)
        o, hT, st_out = _layer_oracle(x[tok], w, cu_r, st[mine], P.g[tok], P.beta[tok], P.h0[mine])
        payload = [None] * world
        dist.all_gather_object(payload, (mine, tok, o, hT, st_out))
        if rank == 0:
            q.put(payload)
    finally:
        dist.destroy_process_group()


def test_layer_sequence_sharding_matches_unsharded():
    """The whole layer prefill (conv windows from each sequence's own state,
    conv, recurrence) shards by sequence the same way: each rank takes its
    sequences' rows of x and rows of the conv state; no exchange is needed."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_layer_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    payload = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, w, cu, st, P = _layer_problem()
    o_ref, h_ref, st_ref = _layer_oracle(x, w, cu, st, P.g, P.beta, P.h0)
    o, hT, sto = (np.full_like(a, np.nan) for a in (o_ref, h_ref, st_ref))
    seen = []
    for mine, tok, o_r, h_r, s_r in payload:
        o[tok] = o_r
        hT[mine] = h_r
        sto[mine] = s_r
        seen += mine
    assert sorted(seen) == list(range(len(cu) - 1))
    assert np.array_equal(o, o_ref) and np.array_equal(hT, h_ref) and np.array_equal(sto, st_ref)


def test_assignment_is_balanced_and_complete():
    lens = [300, 10, 290, 5, 150, 150, 0]
    parts = assign_sequences(lens, 3)
    assert sorted(sum(parts, [])) == list(range(len(lens)))
    loads = [sum(lens[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(lens)
    with pytest.raises(ValueError):
        assign_sequences(lens, 0)
