"""GPU parity of the fused CTA-pair kernel (short side 128 < k <= 256, long
side <= 256): full steps in both orientations, ragged and unaligned shapes,
other iteration counts and coefficients, a call that mixes it with the
single-CTA and the multi-launch paths, and the launch kind it reports."""

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon
from oracle import muon_oracle

from gpu_helpers import REL_BUF, check_band, check_o, gpu_step, o_from_w, relF

pytestmark = pytest.mark.gpu

PAIR_SHAPES = [(256, 256), (200, 256), (256, 200), (129, 130), (130, 129), (256, 129), (250, 251), (131, 256),
               (255, 255)]


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
        W_ref, b_ref, O_ref = muon_oracle.muon_update(W[i], g[i], bufs[i], lr, mu, **kw)
        O = o_from_w(W[i], W_new[i], lr)
        check_o(O, O_ref, f"matrix {i} {W[i].shape}")
        assert relF(b_new[i], b_ref) <= REL_BUF, (i, W[i].shape)
        if band:
            _, G = muon_oracle.momentum_update(g[i], bufs[i], mu, nesterov=kw.get("nesterov", True))
            check_band(O, G)


def test_pair_path_runs_these_shapes():
    muon.profile_enable(True)
    W, g, b = _inputs([(256, 256), (200, 256)], seed=1)
    gpu_step(W, g, b, 0.02, 0.95)
    muon.profile_enable(False)
    prof = muon.profile_read()
    assert prof["pair"][1] == 1 and prof["gram"][1] == 0 and prof["small"][1] == 0


def test_pair_steps_both_orientations_ragged_unaligned():
    W, g, b = _inputs(PAIR_SHAPES, seed=2)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    _check(W, g, b, W_new, b_new)


def test_pair_three_steps_against_oracle():
    shapes = [(256, 256), (180, 240), (240, 180)]
    W, g, b = _inputs(shapes, seed=3)
    dev = torch.device("cuda:0")
    Wd = [torch.from_numpy(x).to(dev) for x in W]
    bd = [torch.from_numpy(x).to(dev) for x in b]
    for step in range(3):
        gs = _inputs(shapes, seed=10 + step)[1]
        W_pre = [x.cpu().numpy() for x in Wd]
        b_pre = [x.cpu().numpy() for x in bd]
        muon.step(Wd, [torch.from_numpy(x).to(dev) for x in gs], bd, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        _check(W_pre, gs, b_pre, [x.cpu().numpy() for x in Wd], [x.cpu().numpy() for x in bd], band=False)


@pytest.mark.parametrize("ns_steps", [0, 1, 2, 6])
def test_pair_other_step_counts(ns_steps):
    for shape in [(240, 256), (256, 240)]:
        gen = torch.Generator().manual_seed(50 + ns_steps)
        G = torch.randn(*shape, generator=gen)
        (O,) = muon.orthogonalize([G.cuda()], ns_steps=ns_steps)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        O_ref = muon_oracle.newton_schulz5(G.numpy().astype(np.float64), steps=ns_steps)
        check_o(O.cpu().numpy(), O_ref, f"{shape} ns_steps={ns_steps}")


def test_pair_plain_momentum_and_custom_coefficients():
    shapes = [(256, 256), (256, 160)]
    W, g, bufs = _inputs(shapes, seed=4)
    W_new, b_new = gpu_step(W, g, bufs, 0.02, 0.9, nesterov=False, a=2.0, b=-1.5, c=0.5)
    _check(W, g, bufs, W_new, b_new, mu=0.9, band=False, nesterov=False, a=2.0, b=-1.5, c=0.5)


def test_pair_mixed_with_small_and_gemm_paths_in_one_call():
    shapes = [(256, 256), (768, 768), (128, 512), (200, 180), (64, 96)]
    W, g, b = _inputs(shapes, seed=5, gscale=0.02)
    muon.profile_enable(True)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    muon.profile_enable(False)
    prof = muon.profile_read()
    assert prof["pair"][1] == 1 and prof["small"][1] == 1 and prof["chain"][1] == 1
    _check(W, g, b, W_new, b_new, band=False)


def test_pair_deterministic_bitwise():
    W, g, b = _inputs([(256, 256), (256, 200)], seed=6)
    r1 = gpu_step(W, g, b, 0.02, 0.95)
    r2 = gpu_step(W, g, b, 0.02, 0.95)
    for x, y in zip(r1[0] + r1[1], r2[0] + r2[1]):
        assert np.array_equal(x, y)
