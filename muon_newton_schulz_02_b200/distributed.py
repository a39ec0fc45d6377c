"""Data-parallel Muon step over several ranks (one process per GPU).

In data-parallel training every rank holds the same weights and, after the
gradient all-reduce, the same gradients (the speedrun context of the
Modded-NanoGPT article trains on 8 GPUs launched with --nproc_per_node).  The
Muon update of each weight matrix is independent of the others, so the ranks
split the matrices: rank r runs the step (momentum, NS5, apply) on the
matrices it owns, then one all_gather gives every rank every updated matrix.
Each rank keeps the momentum buffers of the matrices it owns; the buffers of
other ranks' matrices are left untouched.

Two exchanges: the updated fp32 weights (the owner applies its update in the
step's fused epilogue; 4 bytes per element cross the interconnect), or the
orthogonalised update O in bf16 (2 bytes per element; every rank then applies
every matrix's O itself, so that all replicas of W receive the same bf16
update).

Nothing here loads another GPU's memory directly: the exchange is a NCCL (or,
on the CPU, gloo) all_gather of a packed buffer.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def step_flops(rows: int, cols: int, ns_steps: int = 5) -> float:
    """Algorithmic NS5 flops of one matrix (symmetry of X X^T and A A used)."""
    k, l = min(rows, cols), max(rows, cols)
    return float(ns_steps * (k * (k + 1) * l + k * k * (k + 1) + 2 * k * k * l))


def partition(shapes, world: int, ns_steps: int = 5):
    """Greedy longest-processing-time split: matrices by decreasing flops, each
    to the rank with the least work so far (ties: lowest rank).  Deterministic,
    so every rank computes the same split.  Returns a list of index lists."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-step_flops(*shapes[i], ns_steps), i))
    load = [0.0] * world
    owned = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owned[r].append(i)
        load[r] += step_flops(*shapes[i], ns_steps)
    return [sorted(o) for o in owned]


def _default_local_step(params, grads, bufs, lr, mu, ns_steps):
    from . import step
    step(params, grads, bufs, lr=lr, mu=mu, ns_steps=ns_steps)


def _default_local_update(grads, bufs, O, mu, ns_steps):
    from . import update_bf16
    update_bf16(grads, bufs, mu, ns_steps=ns_steps, O=O)


def _default_local_apply(params, O, lr):
    from . import apply_bf16
    apply_bf16(params, O, lr)


def _padded(n: int) -> int:
    return (n + 7) // 8 * 8              # bf16 slots start 16-byte aligned in the packed buffer


def buckets_of(owned, nbuckets: int):
    """Split every rank's owned indices into `nbuckets` contiguous runs (the
    same count on every rank; a run may be empty)."""
    if nbuckets < 1:
        raise ValueError("nbuckets must be >= 1")
    out = []
    for o in owned:
        q, r = divmod(len(o), nbuckets)
        runs, pos = [], 0
        for j in range(nbuckets):
            n = q + (1 if j < r else 0)
            runs.append(o[pos:pos + n])
            pos += n
        out.append(runs)
    return out


def sharded_step(params, grads, bufs, lr: float, mu: float, ns_steps: int = 5, group=None, local_step=None,
                 nbuckets: int = 1, exchange: str = "w32", local_update=None, local_apply=None):
    """One Muon step split across the ranks of `group` (default: the world).

    params / grads / bufs: the full, identical lists on every rank (same
    device type on all ranks: CUDA with NCCL, CPU with gloo).  On return every
    rank holds every updated matrix.  `local_step(params, grads, bufs, lr, mu,
    ns_steps)` updates a sub-list in place; the default is the CUDA step.

    With nbuckets > 1 each rank's matrices are stepped in that many runs, and
    the all_gather of a finished run is issued asynchronously, so it overlaps
    the step of the next run (every rank issues the same collectives in the
    same order: run j of all ranks goes in the j-th all_gather).

    exchange="o16" sends the bf16 update instead of the fp32 weights:
    `local_update(grads, bufs, O, mu, ns_steps)` writes the owned matrices' O
    (bf16) straight into the packed send buffer, and after each all_gather
    `local_apply(params, O, lr)` applies every matrix of the run on every rank
    (defaults: the CUDA library's update_bf16 / apply_bf16)."""
    if exchange not in ("w32", "o16"):
        raise ValueError("exchange must be 'w32' or 'o16'")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    local_step = local_step or _default_local_step
    shapes = [tuple(p.shape) for p in params]
    owned = partition(shapes, world, ns_steps)
    runs = buckets_of(owned, nbuckets)
    dev = params[0].device
    if exchange == "o16":
        _sharded_o16(params, grads, bufs, lr, mu, ns_steps, group, world, rank, runs, dev,
                     local_update or _default_local_update, local_apply or _default_local_apply)
        return owned
    pending = []
    for j in range(nbuckets):
        mine = runs[rank][j]
        if mine:
            local_step([params[i] for i in mine], [grads[i] for i in mine], [bufs[i] for i in mine], lr, mu, ns_steps)
        if world == 1:
            continue
        chunk = max(sum(params[i].numel() for i in runs[r][j]) for r in range(world))
        if chunk == 0:
            continue                                    # identical on every rank: nobody has a run j
        send = torch.zeros(chunk, dtype=torch.float32, device=dev)
        off = 0
        for i in mine:
            n = params[i].numel()
            send[off:off + n].copy_(params[i].reshape(-1))
            off += n
        recv = [torch.empty(chunk, dtype=torch.float32, device=dev) for _ in range(world)]
        work = dist.all_gather(recv, send, group=group, async_op=nbuckets > 1)
        pending.append((j, recv, work))
    for j, recv, work in pending:
        if work is not None:
            work.wait()
        for r in range(world):
            if r == rank:
                continue
            off = 0
            for i in runs[r][j]:
                n = params[i].numel()
                params[i].reshape(-1).copy_(recv[r][off:off + n])
                off += n
    return owned


def _sharded_o16(params, grads, bufs, lr, mu, ns_steps, group, world, rank, runs, dev, local_update, local_apply):
    """The bf16-update exchange of sharded_step (see there)."""
    def views(buf, idx):
        out, off = [], 0
        for i in idx:
            n = params[i].numel()
            out.append(buf[off:off + n].view(params[i].shape))
            off += _padded(n)
        return out

    pending = []
    for j in range(len(runs[rank])):
        mine = runs[rank][j]
        chunk = max(sum(_padded(params[i].numel()) for i in runs[r][j]) for r in range(world))
        if chunk == 0:
            continue                                    # identical on every rank: nobody has a run j
        send = torch.zeros(chunk, dtype=torch.bfloat16, device=dev)
        if mine:
            local_update([grads[i] for i in mine], [bufs[i] for i in mine], views(send, mine), mu, ns_steps)
        if world == 1:
            local_apply([params[i] for i in mine], views(send, mine), lr)
            continue
        recv = [torch.empty(chunk, dtype=torch.bfloat16, device=dev) for _ in range(world)]
        work = dist.all_gather(recv, send, group=group, async_op=len(runs[rank]) > 1)
        pending.append((j, recv, work))
    for j, recv, work in pending:
        if work is not None:
            work.wait()
        idx = [i for r in range(world) for i in runs[r][j]]
        O = [v for r in range(world) for v in views(recv[r], runs[r][j])]
        if idx:
            local_apply([params[i] for i in idx], O, lr)


def max_over_ranks(value: float, group=None, device=None) -> float:
    """The maximum of a per-rank scalar (timings are reported as the slowest rank)."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
