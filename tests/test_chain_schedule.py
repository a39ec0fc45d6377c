"""The chained launch's work lists, checked on the host (no GPU): every tile of
every phase appears exactly once, each item's `need`
counts exactly the tile halves of the earlier phases of its matrix, and the
lists cannot deadlock -- with every cluster running its list in order and an
item starting only once its matrix's counter reaches `need`, all items finish
whatever the timing (the system is monotone, so running every cluster's head
whenever it is ready reaches the end if and only if no timing can get stuck)."""

import math

import pytest

import muon_newton_schulz_02_b200 as muon

GPT2 = [(768, 768)] * 4 * 12 + [(768, 3072)] * 12 + [(3072, 768)] * 12
SETS = {
    "gpt2_124m": GPT2,
    "square_512": [(512, 512)] * 64,
    "mixed_ragged": [(300, 1000), (1000, 300), (640, 1920), (1600, 1600), (384, 384), (768, 256), (257, 513)],
}


def _tiles(k, l):
    T = math.ceil(math.ceil(k / 128) * 128 / 256)
    Tn = math.ceil(math.ceil(l / 128) * 128 / 256)
    sym = [(i, j) for i in range(T) for j in range(i, T)]
    upd = [(i, j) for i in range(T) for j in range(Tn)]
    return sym, upd


def _fused(r, c):
    k, l = min(r, c), max(r, c)
    return (k <= 128 and math.ceil(l / 64) * 64 <= 512) or (k <= 256 and l <= 256)


@pytest.mark.parametrize("name", sorted(SETS))
@pytest.mark.parametrize("ns_steps", [1, 2, 5])
@pytest.mark.parametrize("nclusters", [1, 3, 74])
def test_lists_cover_every_tile_once_and_cannot_deadlock(name, ns_steps, nclusters):
    shapes = SETS[name]
    items, off = muon.chain_plan(shapes, ns_steps=ns_steps, nclusters=nclusters)
    assert len(off) == nclusters + 1 and off[0] == 0 and off[-1] == len(items)
    assert all(off[c] <= off[c + 1] for c in range(nclusters))
    # coverage and need
    expect = {}
    for m, (r, c) in enumerate(shapes):
        if _fused(r, c):
            continue
        sym, upd = _tiles(min(r, c), max(r, c))
        before = 0
        for j in range(3 * ns_steps):
            it, mode = divmod(j, 3)
            if j == 3 * ns_steps - 1:
                mode = 3                                   # the last update, with W -= lr*O
            for t in (upd if mode >= 2 else sym):
                expect[(m, it, mode) + t] = before
            before += 2 * len(upd if mode >= 2 else sym)
    seen = {}
    for need, m, cls, b, tm, tn, mode, it in items:
        key = (m, it, mode, tm, tn)
        assert key not in seen, f"tile {key} listed twice"
        seen[key] = need
    assert seen == expect
    # one (class, index in class) per matrix and one matrix per (class, index), the
    # classes holding one padded shape each, indices 0.. without gaps: what the
    # bounds-checking build verifies on the device for every item
    slot = {}
    for need, m, cls, b, tm, tn, mode, it in items:
        assert slot.setdefault(m, (cls, b)) == (cls, b), f"matrix {m} under two classes or indices"
    assert len(set(slot.values())) == len(slot)
    by_cls = {}
    for m, (cls, b) in slot.items():
        r, c = shapes[m]
        by_cls.setdefault(cls, {})[b] = (math.ceil(min(r, c) / 128), math.ceil(max(r, c) / 128))
    for cls, members in by_cls.items():
        assert sorted(members) == list(range(len(members))), f"class {cls} indices {sorted(members)}"
        assert len(set(members.values())) == 1, f"class {cls} mixes padded shapes"
    # every cluster runs its list in order; run ready heads until nothing moves
    heads = [off[c] for c in range(nclusters)]
    done = {}
    progress = True
    while progress:
        progress = False
        for c in range(nclusters):
            while heads[c] < off[c + 1]:
                need, m = items[heads[c]][0], items[heads[c]][1]
                if done.get(m, 0) < need:
                    break
                done[m] = done.get(m, 0) + 2
                heads[c] += 1
                progress = True
    assert heads == off[1:], "the work lists can deadlock"


def test_lists_let_the_matrices_finish_together():
    # The lists follow the longest remaining critical path first: every matrix
    # starts early and all of them finish near the end, so the last phases
    # (few tiles each) of many matrices fill the clusters together instead of
    # one long chain running alone at the end.  Judged on the GPT-2-124M set by
    # the positions of the items in the clusters' lists.
    items, off = muon.chain_plan(GPT2, ns_steps=5, nclusters=74)
    first, last = {}, {}
    for c in range(74):
        n = off[c + 1] - off[c]
        for k, (need, m, cls, b, tm, tn, mode, it) in enumerate(items[off[c]:off[c + 1]]):
            if it == 0 and mode == 0:
                first[m] = max(first.get(m, 0.0), k / n)
            if mode == 3:
                last[m] = min(last.get(m, 1.0), k / n)
    assert len(first) == len(last) == len(GPT2)
    assert max(first.values()) < 0.2          # every matrix's first Gram tiles early in the lists
    assert min(last.values()) > 0.8           # every matrix's last update late in the lists
