"""GPU test of muon_step_noalloc, the entry point for callers that cannot
allocate device memory (code inside an allocator or memory-pool callback, or
a process with a fixed device-memory budget).  It must give the same step as
muon_step on two calls in a row, allocate nothing, and refuse requests larger
than its static 64 MiB scratch.  Kept in the last-collected file so that a
run stopping at the first failure has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon

from gpu_helpers import REL_BUF, REL_O, o_from_w, relF

pytestmark = pytest.mark.gpu

SHAPES = [(768, 768)] * 4 + [(768, 3072), (3072, 768), (130, 250), (250, 130)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def test_noalloc_matches_muon_step_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    gen = torch.Generator().manual_seed(77)
    W0 = [torch.randn(*s, generator=gen) * 0.02 for s in SHAPES]
    grads = [[torch.randn(*s, generator=gen) * 0.02 for s in SHAPES] for _ in range(2)]
    Wa = [w.to(dev) for w in W0]
    ba = [torch.zeros_like(w) for w in Wa]
    Wb = [w.to(dev) for w in W0]
    bb = [torch.zeros_like(w) for w in Wb]
    gd = [[g.to(dev) for g in gs] for gs in grads]
    lr, mu = 0.02, 0.95
    muon.step(Wa[:1], gd[0][:1], [torch.zeros_like(Wa[0])], lr=lr, mu=mu)   # library loaded on this device
    torch.cuda.synchronize()
    Wa = [w.to(dev) for w in W0]
    for call in range(2):
        Wa_pre = [w.cpu().numpy() for w in Wa]
        Wb_pre = [w.cpu().numpy() for w in Wb]
        muon.step(Wa, gd[call], ba, lr=lr, mu=mu)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info(dev)
        muon.step_noalloc(Wb, gd[call], bb, lr=lr, mu=mu)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info(dev)
        assert free1 == free0, "muon_step_noalloc changed the free device memory"
        for i in range(len(SHAPES)):
            Oa = o_from_w(Wa_pre[i], Wa[i].cpu().numpy(), lr)
            Ob = o_from_w(Wb_pre[i], Wb[i].cpu().numpy(), lr)
            assert relF(Ob, Oa) <= REL_O, (call, i)
            assert relF(bb[i].cpu().numpy(), ba[i].cpu().numpy()) <= REL_BUF, (call, i)


def _refused(shapes):
    # real device buffers, so that nothing could fault even if a call were accepted
    dev = torch.device("cuda:0")
    ts = [torch.zeros(*s, device=dev) for s in shapes]
    ptrs = (ctypes.c_void_p * len(ts))(*[ctypes.c_void_p(t.data_ptr()) for t in ts])
    sh = (ctypes.c_int64 * (2 * len(shapes)))(*[v for s in shapes for v in s])
    rc = muon.lib().muon_step_noalloc(ptrs, ptrs, ptrs, sh, len(shapes), 0.02, 0.95, 5,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc


def test_noalloc_rejects_requests_beyond_its_scratch():
    assert _refused([(4096, 4096)]) == -7             # needs 4 x 32 MiB of iterates and matrices
    assert "static scratch" in muon.last_error()
    assert _refused([(320, 320)] * 400) == -7         # more matrices than one call takes
    assert _refused([(192, 192)] * 400) == 0          # the CTA-pair kernel needs no scratch
