"""GPU test of muon_step_noalloc, the entry point for callers that cannot
allocate device memory (code inside an allocator or memory-pool callback, or
a process with a fixed device-memory budget).  It runs the same kernels as
muon_step on the same inputs, so its results must be bitwise the same, on two
calls in a row; it must allocate nothing once the library is loaded on the
device, refuse requests larger than its static 64 MiB scratch, and report a
bounded wait that ran out.  Kept in the last-collected file so that a run
stopping at the first failure has already run every other test."""

import ctypes
import os
import subprocess
import sys
import textwrap

import pytest
import torch

import muon_newton_schulz_02_b200 as muon

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(768, 768)] * 4 + [(768, 3072), (3072, 768), (130, 250), (250, 130), (100, 400)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _state(seed):
    gen = torch.Generator().manual_seed(seed)
    W0 = [torch.randn(*s, generator=gen) * 0.02 for s in SHAPES]
    grads = [[torch.randn(*s, generator=gen) * 0.02 for s in SHAPES] for _ in range(3)]
    return W0, grads


def test_noalloc_matches_muon_step_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    W0, grads = _state(77)
    Wa = [w.to(dev) for w in W0]
    ba = [torch.zeros_like(w) for w in Wa]
    Wb = [w.to(dev) for w in W0]
    bb = [torch.zeros_like(w) for w in Wb]
    gd = [[g.to(dev) for g in gs] for gs in grads]
    lr, mu = 0.02, 0.95
    # the library's device code (and with it the static scratch) is loaded on
    # this device by its first call; the calls checked below come after it
    muon.step_noalloc([torch.zeros_like(Wb[0])], gd[0][:1], [torch.zeros_like(Wb[0])], lr=lr, mu=mu)
    torch.cuda.synchronize()
    for call in range(2):
        muon.step(Wa, gd[call], ba, lr=lr, mu=mu)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info(dev)
        muon.step_noalloc(Wb, gd[call], bb, lr=lr, mu=mu)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info(dev)
        assert free1 == free0, "muon_step_noalloc changed the free device memory"
        for i in range(len(SHAPES)):
            assert torch.equal(Wb[i], Wa[i]), f"call {call}: W of matrix {i} {SHAPES[i]} differs from muon_step"
            assert torch.equal(bb[i], ba[i]), f"call {call}: buf of matrix {i} differs from muon_step"


def test_noalloc_first_call_in_a_fresh_process():
    # Where muon_step_noalloc is the library's first call on the device, that
    # call loads the library's device code and with it the 64 MiB array (with
    # CUDA's lazy module loading); the next call allocates nothing.  Both calls
    # give muon_step's result.
    code = textwrap.dedent("""
        import sys, torch
        sys.path.insert(0, %r)
        import muon_newton_schulz_02_b200 as muon
        dev = torch.device("cuda:0")
        torch.cuda.init()
        gen = torch.Generator().manual_seed(5)
        shapes = [(768, 768), (768, 3072)]
        W = [(torch.randn(*s, generator=gen) * 0.02).to(dev) for s in shapes]
        g = [(torch.randn(*s, generator=gen) * 0.02).to(dev) for s in shapes]
        b = [torch.zeros_like(x) for x in W]
        W2 = [x.clone() for x in W]; b2 = [x.clone() for x in b]
        torch.cuda.synchronize()
        f0 = torch.cuda.mem_get_info(dev)[0]
        muon.step_noalloc(W, g, b, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        f1 = torch.cuda.mem_get_info(dev)[0]
        muon.step_noalloc(W, g, b, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        f2 = torch.cuda.mem_get_info(dev)[0]
        for _ in range(2):
            muon.step(W2, g, b2, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        same = all(torch.equal(x, y) for x, y in zip(W + b, W2 + b2))
        print("FIRST_CALL_BYTES", f0 - f1, "SECOND_CALL_BYTES", f1 - f2, "SAME", int(same))
    """ % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = [x for x in out.stdout.splitlines() if x.startswith("FIRST_CALL_BYTES")][-1].split()
    first, second, same = int(line[1]), int(line[3]), int(line[5])
    print(f"free device memory taken by the first call: {first} bytes; by the second: {second}")
    assert second == 0, f"the second call changed the free device memory by {second} bytes"
    assert 0 <= first <= (128 << 20), f"the first call took {first} bytes (module load expected: ~64 MiB + code)"
    assert same == 1, "muon_step_noalloc differs from muon_step"


def test_noalloc_reports_a_bounded_wait_that_ran_out():
    dev = torch.device("cuda:0")
    W0, grads = _state(78)
    shapes_gemm = SHAPES[:6]                       # matrices that run through the phase launches
    n = len(shapes_gemm)
    Wa = [w.to(dev) for w in W0[:n]]
    ba = [torch.zeros_like(w) for w in Wa]
    Wb = [w.to(dev) for w in W0[:n]]
    bb = [torch.zeros_like(w) for w in Wb]
    g = [x.to(dev) for x in grads[0][:n]]
    muon.debug_set(1, 20_000_000)                  # next GEMM launch skips a pipeline fill; 20 ms bound
    try:
        muon.step_noalloc([w.clone() for w in Wb], g, [b.clone() for b in bb], lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        with pytest.raises(muon.MuonError) as ei:  # the next call reports it and launches nothing
            muon.step_noalloc(Wb, g, bb, lr=0.02, mu=0.95)
        assert ei.value.code == -5 and "bounded wait" in str(ei.value)
    finally:
        muon.debug_set(0, 0)
    muon.step_noalloc(Wb, g, bb, lr=0.02, mu=0.95)  # the context survived and the call runs again
    muon.step(Wa, g, ba, lr=0.02, mu=0.95)
    torch.cuda.synchronize()
    for x, y in zip(Wa + ba, Wb + bb):
        assert torch.equal(x, y)


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
