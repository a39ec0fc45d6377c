"""GPU parity of the fused four-CTA kernel (short side k <= 128, long side
256 < l <= 512, at most 37 such matrices in a call): steps in both
orientations, ragged and unaligned shapes, other iteration counts,
coefficients and plain momentum, NS5 alone, determinism, the launch kind it
reports, and the switch back to one CTA per matrix for larger batches."""

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon
from oracle import muon_oracle

from gpu_helpers import REL_BUF, check_band, check_o, gpu_step, o_from_w, relF

pytestmark = pytest.mark.gpu

QUAD_SHAPES = [(128, 512), (512, 128), (100, 300), (300, 100), (128, 400), (7, 260), (1, 511), (511, 1),
               (97, 385), (64, 257)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _inputs(shapes, seed, gscale=1.0, bscale=0.1):
    gen = torch.Generator().manual_seed(seed)
    W = [(torch.randn(*s, generator=gen) * 0.02).numpy() for s in shapes]
    g = [(torch.randn(*s, generator=gen) * gscale).numpy() for s in shapes]
    b = [(torch.randn(*s, generator=gen) * bscale).numpy() for s in shapes]
    return W, g, b


def _check(W, g, bufs, W_new, b_new, lr=0.02, mu=0.95, band=True, **kw):
    for i in range(len(W)):
        _, b_ref, O_ref = muon_oracle.muon_update(W[i], g[i], bufs[i], lr, mu, **kw)
        O = o_from_w(W[i], W_new[i], lr)
        check_o(O, O_ref, f"matrix {i} {W[i].shape}")
        assert relF(b_new[i], b_ref) <= REL_BUF, (i, W[i].shape)
        if band and min(W[i].shape) > 1:
            _, G = muon_oracle.momentum_update(g[i], bufs[i], mu, nesterov=kw.get("nesterov", True))
            check_band(O, G)


def _kinds(shapes, seed=1):
    muon.profile_enable(True)
    muon.profile_read()
    W, g, b = _inputs(shapes, seed)
    gpu_step(W, g, b, 0.02, 0.95)
    muon.profile_enable(False)
    return muon.profile_read()


def test_quad_path_runs_a_few_long_small_matrices():
    prof = _kinds([(128, 512), (512, 128), (100, 200)])
    assert prof["quad"][1] == 1 and prof["small"][1] == 1 and prof["gram"][1] == 0
    prof = _kinds([(128, 512)] * 40)              # a full batch: one CTA per matrix instead
    assert prof["quad"][1] == 0 and prof["small"][1] == 1


def test_quad_steps_both_orientations_ragged():
    W, g, b = _inputs(QUAD_SHAPES, seed=2)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    _check(W, g, b, W_new, b_new)


def test_quad_and_single_cta_paths_agree_with_the_oracle_on_the_same_matrix():
    shapes = [(128, 512)]
    W, g, b = _inputs(shapes, seed=3)
    quad, _ = gpu_step(W, g, b, 0.02, 0.95)
    # the same matrix in a batch of 38, which takes the single-CTA kernel
    single, _ = gpu_step(W * 38, g * 38, b * 38, 0.02, 0.95)
    _, _, O_ref = muon_oracle.muon_update(W[0], g[0], b[0], 0.02, 0.95)
    for got, what in ((quad[0], "quad"), (single[0], "single"), (single[37], "single, last")):
        check_o(o_from_w(W[0], got, 0.02), O_ref, what)


@pytest.mark.parametrize("ns_steps", [0, 1, 2, 6])
def test_quad_other_step_counts(ns_steps):
    shapes = [(128, 512), (300, 100)]
    W, g, b = _inputs(shapes, seed=4)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95, ns_steps=ns_steps)
    _check(W, g, b, W_new, b_new, band=False, steps=ns_steps)


def test_quad_coefficients_and_plain_momentum():
    shapes = [(128, 512), (400, 90)]
    W, g, b = _inputs(shapes, seed=5)
    kw = dict(a=2.0, b=-1.5, c=0.5, nesterov=False)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.9, **kw)
    _check(W, g, b, W_new, b_new, mu=0.9, band=False, **kw)


def test_quad_orthogonalize_alone():
    shapes = [(128, 512), (512, 100)]
    gen = torch.Generator().manual_seed(6)
    G = [torch.randn(*s, generator=gen) for s in shapes]
    O = muon.orthogonalize([x.cuda() for x in G])
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        check_o(O[i].cpu().numpy(), muon_oracle.newton_schulz5(G[i].numpy()), f"{shapes[i]}")


def test_quad_deterministic_and_unaligned():
    shapes = [(128, 512), (300, 77)]
    W, g, b = _inputs(shapes, seed=7)
    r1, b1 = gpu_step(W, g, b, 0.02, 0.95)
    r2, b2 = gpu_step(W, g, b, 0.02, 0.95)
    for i in range(len(shapes)):
        assert np.array_equal(r1[i], r2[i]) and np.array_equal(b1[i], b2[i])
    # views that start 1 float into their storage: not 16-byte aligned
    dev = torch.device("cuda:0")

    def mis(a):
        t = torch.empty(a.size + 1, device=dev)
        v = t[1:].view(*a.shape)
        v.copy_(torch.as_tensor(a))
        return v
    Wd, gd, bd = [mis(x) for x in W], [mis(x) for x in g], [mis(x) for x in b]
    muon.step(Wd, gd, bd, lr=0.02, mu=0.95)
    torch.cuda.synchronize()
    assert muon.sync_status() == 0, muon.last_error()
    _check(W, g, b, [x.cpu().numpy() for x in Wd], [x.cpu().numpy() for x in bd])


def test_quad_bounded_wait_timeout_is_reported_and_context_survives():
    shapes = [(128, 512), (300, 100)]
    W, g, b = _inputs(shapes, seed=8)
    dev = torch.device("cuda:0")
    Wd = [torch.as_tensor(x).to(dev) for x in W]
    gd = [torch.as_tensor(x).to(dev) for x in g]
    bd = [torch.as_tensor(x).to(dev) for x in b]
    # the next four-CTA launch keeps back one CTA's first Gram partial: the owner's
    # wait for it runs out, then every other CTA's wait for the owner's rows of A
    muon.debug_set(8, 20_000_000)
    try:
        muon.step(Wd, gd, bd, lr=0.02, mu=0.95)
        assert muon.sync_status() == -5               # MUON_ERR_TIMEOUT
        assert "bounded wait" in muon.last_error()
    finally:
        muon.debug_set(0, 0)
    # the context is still usable and the next step is right
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    _check(W, g, b, W_new, b_new)


@pytest.mark.parametrize("count,kind", [(37, "quad"), (38, "small")])
def test_quad_batch_limit(count, kind):
    # 37 clusters of four CTAs fill one wave of 148 SMs; one matrix more takes
    # the single-CTA kernel for the whole batch
    shapes = [(128, 512) if i % 2 == 0 else (300, 96) for i in range(count)]
    muon.profile_enable(True)
    muon.profile_read()
    W, g, b = _inputs(shapes, seed=9)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    muon.profile_enable(False)
    prof = muon.profile_read()
    assert prof[kind][1] == 1 and prof["quad" if kind == "small" else "small"][1] == 0
    sub = [0, 1, count // 2, count - 1]
    _check([W[i] for i in sub], [g[i] for i in sub], [b[i] for i in sub],
           [W_new[i] for i in sub], [b_new[i] for i in sub])
