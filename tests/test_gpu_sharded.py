"""The data-parallel sharded step driving the real CUDA step: two gloo ranks
(processes) share cuda:0, each runs muon.step on the matrices it owns, and the
exchange goes through host copies (gloo all_gather of CPU tensors).  Every rank
must end with every updated matrix, bitwise equal to one process stepping all
matrices on the GPU, and within the parity bar of the oracle.  The two
processes' kernels are independent: nothing waits on the other rank's GPU
work."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gpu_helpers import REL_BUF, check_o, o_from_w, relF

pytestmark = pytest.mark.gpu

SHAPES = [(768, 768)] * 3 + [(768, 3072), (3072, 768), (256, 200), (100, 300), (640, 384)]


def _inputs():
    gen = torch.Generator().manual_seed(123)
    W = [torch.randn(*s, generator=gen) * 0.02 for s in SHAPES]
    g = [torch.randn(*s, generator=gen) * 0.02 for s in SHAPES]
    b = [torch.randn(*s, generator=gen) * 0.01 for s in SHAPES]
    return W, g, b


def _cuda_local_step(params, grads, bufs, lr, mu, ns_steps):
    import muon_newton_schulz_02_b200 as muon
    dev = torch.device("cuda:0")
    Wd = [x.to(dev) for x in params]
    gd = [x.to(dev) for x in grads]
    bd = [x.to(dev) for x in bufs]
    muon.step(Wd, gd, bd, lr=lr, mu=mu, ns_steps=ns_steps)
    torch.cuda.synchronize()
    assert muon.sync_status() == 0, muon.last_error()
    for h, d in zip(params + bufs, Wd + bd):
        h.copy_(d.cpu())


def _worker(rank, world, port, nbuckets, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from muon_newton_schulz_02_b200 import distributed as mdist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, g, b = _inputs()
        owned = mdist.sharded_step(W, g, b, lr=0.02, mu=0.95, local_step=_cuda_local_step, nbuckets=nbuckets)
        q.put((rank, [w.numpy() for w in W], [x.numpy() for x in b], owned))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("nbuckets", [1, 2])
def test_sharded_step_with_the_cuda_step_on_two_ranks(nbuckets):
    import __graft_entry__
    __graft_entry__.build()
    from oracle import muon_oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, nbuckets, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=600) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    W0, g0, b0 = _inputs()
    W1, b1 = [x.clone() for x in W0], [x.clone() for x in b0]
    _cuda_local_step(W1, g0, b1, 0.02, 0.95, 5)                # one process, every matrix
    partition = results[0][3]                                  # the same split on both ranks
    assert sorted(i for o in partition for i in o) == list(range(len(SHAPES)))
    for rank, W, b, owned in results:
        assert owned == partition
        for i in range(len(SHAPES)):
            assert np.array_equal(W[i], W1[i].numpy()), (rank, i)
        for i in owned[rank]:
            assert np.array_equal(b[i], b1[i].numpy()), (rank, i)
    for i in (0, 3, 4, 5, 7):
        W_ref, b_ref, O_ref = muon_oracle.muon_update(W0[i].numpy(), g0[i].numpy(), b0[i].numpy(), 0.02, 0.95)
        check_o(o_from_w(W0[i].numpy(), results[0][1][i], 0.02), O_ref, f"matrix {i} {SHAPES[i]}")
        owner = [r for r in range(2) if i in partition[r]][0]
        b_owner = [b for r, _, b, _ in results if r == owner][0]
        assert relF(b_owner[i], b_ref) <= REL_BUF


# ---- the bf16-update exchange with the CUDA library's two halves -----------
def _cuda_local_update(grads, bufs, O, mu, ns_steps):
    import muon_newton_schulz_02_b200 as muon
    dev = torch.device("cuda:0")
    gd = [x.to(dev) for x in grads]
    bd = [x.to(dev) for x in bufs]
    Od = [torch.empty(o.shape, dtype=torch.bfloat16, device=dev) for o in O]
    muon.update_bf16(gd, bd, mu, ns_steps=ns_steps, O=Od)
    torch.cuda.synchronize()
    assert muon.sync_status() == 0, muon.last_error()
    for h, d in zip(bufs + O, bd + Od):
        h.copy_(d.cpu())


def _cuda_apply(params, O, lr):
    import muon_newton_schulz_02_b200 as muon
    dev = torch.device("cuda:0")
    Wd = [x.to(dev) for x in params]
    muon.apply_bf16(Wd, [o.to(dev) for o in O], lr)
    torch.cuda.synchronize()
    for h, d in zip(params, Wd):
        h.copy_(d.cpu())


def _worker_o16(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from muon_newton_schulz_02_b200 import distributed as mdist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, g, b = _inputs()
        owned = mdist.sharded_step(W, g, b, lr=0.02, mu=0.95, nbuckets=2, exchange="o16",
                                   local_update=_cuda_local_update, local_apply=_cuda_apply)
        q.put((rank, [w.numpy() for w in W], [x.numpy() for x in b], owned))
    finally:
        dist.destroy_process_group()


def test_bf16_update_exchange_with_the_cuda_halves_on_two_ranks():
    import __graft_entry__
    __graft_entry__.build()
    from oracle import muon_oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_o16, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=600) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    W0, g0, b0 = _inputs()
    partition = results[0][3]
    for i in range(len(SHAPES)):
        assert np.array_equal(results[0][1][i], results[1][1][i]), i      # identical replicas
    for i in range(len(SHAPES)):
        W_ref, b_ref, O_ref = muon_oracle.muon_update(W0[i].numpy(), g0[i].numpy(), b0[i].numpy(), 0.02, 0.95)
        check_o(o_from_w(W0[i].numpy(), results[0][1][i], 0.02), O_ref, f"matrix {i} {SHAPES[i]}")
        owner = [r for r in range(2) if i in partition[r]][0]
        b_owner = [b for r, _, b, _ in results if r == owner][0]
        assert relF(b_owner[i], b_ref) <= REL_BUF
