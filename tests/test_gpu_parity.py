"""GPU parity: the CUDA path (through the C ABI) against the CPU fp64 oracle on
the same seeded inputs.  Bar: relF(O) <= 3e-2, momentum buffer <= 1e-6
relative, singular values of O in the band (see gpu_helpers)."""

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


def test_single_128x512_step():
    w = workloads.get("single_128x512")
    g = workloads.grad(w, 0, 0).numpy()
    W = workloads.weight(w, 0).numpy()
    buf = np.zeros_like(g)
    (W_new,), (b_new,) = gpu_step([W], [g], [buf], w.lr, w.mu)
    W_ref, b_ref, O_ref = muon_oracle.muon_update(W, g, buf, w.lr, w.mu)
    O = o_from_w(W, W_new, w.lr)
    check_o(O, O_ref, "single_128x512")
    assert relF(b_new, b_ref) <= REL_BUF
    assert np.abs(b_new - b_ref).max() <= REL_BUF * np.abs(b_ref).max()
    _, G = muon_oracle.momentum_update(g, buf, w.mu)
    check_band(O, G)


SHAPES = [(128, 512), (512, 128), (128, 128), (256, 384), (384, 256), (768, 768), (640, 1920),
          (127, 129), (129, 127), (300, 1000), (1000, 300), (1, 1), (1, 7), (7, 1), (3, 5), (33, 65),
          (200, 200), (1600, 1600)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{r}x{c}" for r, c in SHAPES])
def test_orthogonalize_shapes(shape):
    gen = torch.Generator().manual_seed(hash(shape) % 2**31)
    G = torch.randn(*shape, generator=gen)
    (O,) = muon.orthogonalize([G.cuda()])
    torch.cuda.synchronize()
    assert muon.sync_status() == 0
    O_ref = muon_oracle.newton_schulz5(G.numpy().astype(np.float64))
    check_o(O.cpu().numpy(), O_ref, str(shape))


def test_orthogonalize_batch_mixed_shapes():
    shapes = [(768, 768)] * 3 + [(768, 3072), (3072, 768), (130, 70), (70, 130)]
    gen = torch.Generator().manual_seed(5)
    Gs = [torch.randn(*s, generator=gen) * 0.02 for s in shapes]
    Os = muon.orthogonalize([g.cuda() for g in Gs])
    torch.cuda.synchronize()
    for g, o in zip(Gs, Os):
        O_ref = muon_oracle.newton_schulz5(g.numpy().astype(np.float64))
        check_o(o.cpu().numpy(), O_ref, str(tuple(g.shape)))


@pytest.mark.parametrize("ns_steps", [0, 1, 2, 7])
def test_other_step_counts(ns_steps):
    gen = torch.Generator().manual_seed(40 + ns_steps)
    G = torch.randn(256, 640, generator=gen)
    (O,) = muon.orthogonalize([G.cuda()], ns_steps=ns_steps)
    torch.cuda.synchronize()
    O_ref = muon_oracle.newton_schulz5(G.numpy().astype(np.float64), steps=ns_steps)
    check_o(O.cpu().numpy(), O_ref, f"ns_steps={ns_steps}")
