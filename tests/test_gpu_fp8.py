"""GPU tests of the reduced-precision variant muon_step_fp8 (e4m3 operands in
the first one or two Newton-Schulz iterations, in the launches that run one
phase each): parity with the fp64 oracle at the same bar as the bf16 path on
every workload (those that normally run in the chained launch are run here with
one launch per phase, so that they take the e4m3 products), the chained groups
keeping bf16 operands, determinism, the iteration-count and coefficient edge
cases, and fp8_iters = 0 being the bf16 step itself."""

import contextlib

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon
from muon_newton_schulz_02_b200 import workloads
from oracle import muon_oracle

from gpu_helpers import REL_BUF, check_band, check_o, gpu_step, o_from_w, relF

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _inputs(shapes, seed):
    gen = torch.Generator().manual_seed(seed)
    W = [(torch.randn(*s, generator=gen) * 0.02).numpy() for s in shapes]
    g = [torch.randn(*s, generator=gen).numpy() for s in shapes]
    b = [(torch.randn(*s, generator=gen) * 0.1).numpy() for s in shapes]
    return W, g, b


@contextlib.contextmanager
def per_phase():
    """One launch per phase for every group (where the e4m3 products run)."""
    muon.debug_set(4)
    try:
        yield
    finally:
        muon.debug_set(0)


def _workload_errors(name, fp8_iters, subset, band_subset=(), steps=1, svd_device="cpu"):
    """Runs the whole workload with muon_step_fp8 and checks the subset against
    the oracle at the parity bar; returns the subset's relF errors."""
    w = workloads.get(name)
    dev = torch.device("cuda:0")
    W = workloads.weights(w, device=dev)
    bufs = workloads.zero_bufs(w, device=dev)
    errs = []
    for step in range(steps):
        g = workloads.grads(w, step, device=dev)
        W_pre = {i: W[i].cpu().numpy() for i in subset}
        b_pre = {i: bufs[i].cpu().numpy() for i in subset}
        g_h = {i: g[i].cpu().numpy() for i in subset}
        muon.step(W, g, bufs, lr=w.lr, mu=w.mu, fp8_iters=fp8_iters)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        for i in subset:
            _, b_ref, O_ref = muon_oracle.muon_update(W_pre[i], g_h[i], b_pre[i], w.lr, w.mu)
            O = o_from_w(W_pre[i], W[i].cpu().numpy(), w.lr)
            err, _ = check_o(O, O_ref, f"{name} fp8_iters={fp8_iters} step {step} matrix {i} {w.shapes[i]}")
            errs.append(err)
            assert relF(bufs[i].cpu().numpy(), b_ref) <= REL_BUF
            if i in band_subset and step == 0:
                _, G = muon_oracle.momentum_update(g_h[i], b_pre[i], w.mu)
                check_band(O, G, svd_device=svd_device)
        del g
    del W, bufs
    torch.cuda.empty_cache()
    return errs


@pytest.mark.parametrize("fp8_iters", [1, 2])
def test_gpt2_124m(fp8_iters):
    # 768x768, 768x3072, 3072x768 of the first layer and the last matrix of the set
    with per_phase():
        _workload_errors("gpt2_124m", fp8_iters, [0, 4, 5, 71], band_subset=[0, 4], steps=2)


@pytest.mark.parametrize("n", [512, 1024, 2048])
def test_square_batches(n):
    with per_phase():
        _workload_errors(f"square_n{n}", 2, [0, 63], band_subset=[0])


def test_square_n4096_last_matrix():
    _workload_errors("square_n4096", 2, [63], band_subset=[63], svd_device="cuda:0")


def test_gpt2_xl_one_step():
    # short side 1600: one launch per phase carries the e4m3 products
    _workload_errors("gpt2_xl_1p5b", 2, [0, 4, 5], band_subset=[0])


def test_illconditioned_and_tall():
    with per_phase():
        _workload_errors("illcond_1024x4096", 2, [0, 15], band_subset=[0, 15])
        _workload_errors("tall_8192x1024", 2, [0, 15], band_subset=[0])


def test_single_128x512_keeps_bf16_operands():
    # a matrix the single-CTA kernel runs whole: the variant is the bf16 step
    W, g, b = _inputs([(128, 512)], 3)
    W0, b0 = gpu_step(W, g, b, 0.02, 0.95)
    W1, b1 = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2)
    assert np.array_equal(W0[0], W1[0]) and np.array_equal(b0[0], b1[0])


def test_zero_fp8_iters_is_the_bf16_step():
    shapes = [(768, 3072), (3072, 768), (1024, 1024)]
    W, g, b = _inputs(shapes, 4)
    W0, b0 = gpu_step(W, g, b, 0.02, 0.95)
    dev = torch.device("cuda:0")
    Wd = [torch.as_tensor(x).to(dev) for x in W]
    gd = [torch.as_tensor(x).to(dev) for x in g]
    bd = [torch.as_tensor(x).to(dev) for x in b]
    pp, gp, bp, sh, n = muon._marshal_step(Wd, gd, bd)
    rc = muon.lib().muon_step_fp8(pp, gp, bp, sh, n, 0.02, 0.95, 5, muon.NS_A, muon.NS_B, muon.NS_C, muon.NS_EPS,
                                  1, 0, None)
    assert rc == 0, muon.last_error()
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert np.array_equal(Wd[i].cpu().numpy(), W0[i])


def test_chained_groups_keep_bf16_operands_and_per_phase_groups_do_not():
    chained = [(768, 3072), (3072, 768), (768, 768), (1024, 1280), (384, 900), (700, 300)]
    W, g, b = _inputs(chained, 5)
    ref, _ = gpu_step(W, g, b, 0.02, 0.95)
    got, _ = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2)
    for i in range(len(chained)):
        assert np.array_equal(got[i], ref[i]), chained[i]
    large = [(1100, 2000), (2000, 1100)]            # short side above 1024: one launch per phase
    W, g, b = _inputs(large, 9)
    ref, _ = gpu_step(W, g, b, 0.02, 0.95)
    got, _ = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2)
    for i in range(len(large)):
        assert not np.array_equal(got[i], ref[i]), large[i]      # the e4m3 products ran
        _, _, O_ref = muon_oracle.muon_update(W[i], g[i], b[i], 0.02, 0.95)
        check_o(o_from_w(W[i], got[i], 0.02), O_ref, f"{large[i]}")


def test_deterministic_and_ragged():
    shapes = [(300, 700), (700, 300), (1000, 300), (260, 1030), (1100, 2000)]
    W, g, b = _inputs(shapes, 6)
    with per_phase():
        r1, b1 = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2)
        r2, _ = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2)
    for i in range(len(shapes)):
        assert np.array_equal(r1[i], r2[i]), shapes[i]
        _, b_ref, O_ref = muon_oracle.muon_update(W[i], g[i], b[i], 0.02, 0.95)
        check_o(o_from_w(W[i], r1[i], 0.02), O_ref, f"{shapes[i]}")
        assert relF(b1[i], b_ref) <= REL_BUF


@pytest.mark.parametrize("ns_steps", [1, 2, 3])
def test_few_iterations(ns_steps):
    # fp8_iters is capped at ns_steps; with 1 or 2 steps the e4m3 products
    # reach the last iteration, whose update writes W
    shapes = [(768, 3072), (512, 512)]
    W, g, b = _inputs(shapes, 7)
    with per_phase():
        Wn, _ = gpu_step(W, g, b, 0.02, 0.95, ns_steps=ns_steps, fp8_iters=2)
    for i in range(len(shapes)):
        _, _, O_ref = muon_oracle.muon_update(W[i], g[i], b[i], 0.02, 0.95, steps=ns_steps)
        check_o(o_from_w(W[i], Wn[i], 0.02), O_ref, f"{shapes[i]} ns_steps={ns_steps}")


def test_other_coefficients():
    # the cubic (2, -1.5, 0.5): other bounds, so other power-of-two scales
    shapes = [(768, 3072), (1024, 1024)]
    W, g, b = _inputs(shapes, 8)
    kw = dict(a=2.0, b=-1.5, c=0.5)
    with per_phase():
        Wn, _ = gpu_step(W, g, b, 0.02, 0.95, fp8_iters=2, **kw)
    for i in range(len(shapes)):
        _, _, O_ref = muon_oracle.muon_update(W[i], g[i], b[i], 0.02, 0.95, **kw)
        check_o(o_from_w(W[i], Wn[i], 0.02), O_ref, f"{shapes[i]} cubic")


def test_rejects_more_than_two_iterations():
    dev = torch.device("cuda:0")
    W = [torch.zeros(768, 768, device=dev)]
    with pytest.raises(muon.MuonError):
        muon.step(W, [torch.ones_like(W[0])], [torch.zeros_like(W[0])], lr=0.02, mu=0.95, fp8_iters=3)
