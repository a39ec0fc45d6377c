"""Multi-rank host logic on the CPU with the gloo backend (world size 2 and 3):
the flop-balanced partition, the sharded step's exchange (every rank ends with
every updated matrix, equal to a single-process step; in one all_gather or in
several asynchronous ones overlapping the step), and the max-over-ranks timing
reduction.  The per-rank compute is injected: here the CPU oracle stands
in for the CUDA step, which needs a GPU."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from muon_newton_schulz_02_b200 import distributed as mdist

SHAPES = [(768, 768)] * 4 + [(768, 3072), (3072, 768), (64, 96), (96, 64), (128, 128)]


def test_partition_covers_each_matrix_once_and_balances():
    for world in (1, 2, 3, 8):
        owned = mdist.partition(SHAPES, world)
        flat = sorted(i for o in owned for i in o)
        assert flat == list(range(len(SHAPES)))
        loads = [sum(mdist.step_flops(*SHAPES[i]) for i in o) for o in owned]
        biggest = max(mdist.step_flops(*s) for s in SHAPES)
        assert max(loads) - min(loads) <= biggest          # LPT bound
    assert mdist.partition(SHAPES, 2) == mdist.partition(SHAPES, 2)   # deterministic


def _oracle_local_step(params, grads, bufs, lr, mu, ns_steps):
    from oracle import muon_oracle
    for W, g, b in zip(params, grads, bufs):
        W_new, b_new, _ = muon_oracle.muon_update(W.numpy(), g.numpy(), b.numpy(), lr, mu, steps=ns_steps)
        W.copy_(torch.from_numpy(W_new))
        b.copy_(torch.from_numpy(b_new))


def _inputs(seed=3, shapes=SHAPES):
    gen = torch.Generator().manual_seed(seed)
    W = [torch.randn(*s, generator=gen) * 0.02 for s in shapes]
    g = [torch.randn(*s, generator=gen) * 0.02 for s in shapes]
    b = [torch.randn(*s, generator=gen) * 0.01 for s in shapes]
    return W, g, b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shapes, q, nbuckets=1):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, g, b = _inputs(shapes=shapes)
        owned = mdist.sharded_step(W, g, b, lr=0.02, mu=0.95, local_step=_oracle_local_step, nbuckets=nbuckets)
        t = mdist.max_over_ranks(float(rank) + 0.5)
        q.put((rank, [w.numpy() for w in W], [x.numpy() for x in b], owned, t))
    finally:
        dist.destroy_process_group()


def test_buckets_split_each_rank_into_runs():
    owned = mdist.partition(SHAPES, 3)
    for nb in (1, 2, 4, 7):
        runs = mdist.buckets_of(owned, nb)
        for o, rr in zip(owned, runs):
            assert len(rr) == nb and [i for run in rr for i in run] == o
            assert max(map(len, rr)) - min(map(len, rr)) <= 1
    with pytest.raises(ValueError):
        mdist.buckets_of(owned, 0)


@pytest.mark.parametrize("world,nbuckets", [(2, 1), (3, 1), (2, 3), (3, 4)])
def test_sharded_step_matches_single_process(world, nbuckets):
    shapes = SHAPES[4:]                                  # keep the CPU oracle quick
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shapes, q, nbuckets)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W_ref, g_ref, b_ref = _inputs(shapes=shapes)
    _oracle_local_step(W_ref, g_ref, b_ref, 0.02, 0.95, 5)
    for rank, W, b, owned, t in results:
        assert t == world - 1 + 0.5                       # max over ranks
        for i in range(len(shapes)):
            assert np.array_equal(W[i], W_ref[i].numpy()), (rank, i)   # every rank has every update
        for i in owned[rank]:
            assert np.array_equal(b[i], b_ref[i].numpy()), (rank, i)   # own momentum updated


# ---- the bf16-update exchange: the owner computes O, every rank applies it --
def _oracle_local_update(grads, bufs, O, mu, ns_steps):
    from oracle import muon_oracle
    for g, b, o in zip(grads, bufs, O):
        b_new, G = muon_oracle.momentum_update(g.numpy(), b.numpy(), mu)
        o.copy_(torch.from_numpy(muon_oracle.newton_schulz5(G, steps=ns_steps)).to(torch.bfloat16))
        b.copy_(torch.from_numpy(b_new))


def _cpu_apply(params, O, lr):
    for W, o in zip(params, O):
        W.sub_(o.float() * lr)


def _worker_o16(rank, world, port, shapes, q, nbuckets):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, g, b = _inputs(shapes=shapes)
        owned = mdist.sharded_step(W, g, b, lr=0.02, mu=0.95, nbuckets=nbuckets, exchange="o16",
                                   local_update=_oracle_local_update, local_apply=_cpu_apply)
        q.put((rank, [w.numpy() for w in W], [x.numpy() for x in b], owned))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,nbuckets", [(2, 1), (3, 2)])
def test_bf16_update_exchange_gives_every_rank_the_same_weights(world, nbuckets):
    shapes = SHAPES[4:]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_o16, args=(r, world, port, shapes, q, nbuckets)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # one process doing the same: update every matrix, then apply every bf16 O
    W_ref, g_ref, b_ref = _inputs(shapes=shapes)
    O = [torch.empty(s, dtype=torch.bfloat16) for s in shapes]
    _oracle_local_update(g_ref, b_ref, O, 0.95, 5)
    _cpu_apply(W_ref, O, 0.02)
    for rank, W, b, owned in results:
        for i in range(len(shapes)):
            assert np.array_equal(W[i], W_ref[i].numpy()), (rank, i)
        for i in owned[rank]:
            assert np.array_equal(b[i], b_ref[i].numpy()), (rank, i)
    with pytest.raises(ValueError):
        mdist.sharded_step(W_ref, g_ref, b_ref, 0.02, 0.95, exchange="fp8")
