"""GPU tests of the full Muon step through the C ABI: the fused apply in both
orientations, ragged and misaligned matrices, method variants, grouping
limits, determinism, checkpoint/resume, the host-buffer entry point and
bounded-wait fault injection (made on the host; nothing faults the GPU)."""

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


def _inputs(shapes, seed, gscale=1.0, bscale=0.1):
    gen = torch.Generator().manual_seed(seed)
    W = [(torch.randn(*s, generator=gen) * 0.02).numpy() for s in shapes]
    g = [(torch.randn(*s, generator=gen) * gscale).numpy() for s in shapes]
    b = [(torch.randn(*s, generator=gen) * bscale).numpy() for s in shapes]
    return W, g, b


def _check_step(W, g, bufs, W_new, b_new, lr=0.02, mu=0.95, **kw):
    for i in range(len(W)):
        W_ref, b_ref, O_ref = muon_oracle.muon_update(W[i], g[i], bufs[i], lr, mu, **kw)
        check_o(o_from_w(W[i], W_new[i], lr), O_ref, f"matrix {i} {W[i].shape}")
        assert relF(b_new[i], b_ref) <= REL_BUF, f"buf {i}"


STEP_SHAPES = [(256, 768), (768, 256), (130, 250), (250, 130), (64, 2000), (2000, 64), (5, 3), (3, 5), (1, 300)]


def test_step_apply_both_orientations_and_ragged():
    W, g, b = _inputs(STEP_SHAPES, 1)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    _check_step(W, g, b, W_new, b_new)


def test_step_misaligned_pointers():
    # views that start 1 float into their storage: not 16-byte aligned
    shapes = [(96, 200), (200, 96)]
    W, g, b = _inputs(shapes, 2)
    dev = torch.device("cuda:0")

    def mis(a):
        t = torch.empty(a.size + 1, device=dev)
        v = t[1:].view(*a.shape)
        v.copy_(torch.as_tensor(a))
        return v
    Wd, gd, bd = [mis(x) for x in W], [mis(x) for x in g], [mis(x) for x in b]
    assert all(t.data_ptr() % 16 for t in Wd)
    muon.step(Wd, gd, bd, lr=0.02, mu=0.95)
    torch.cuda.synchronize()
    _check_step(W, g, b, [t.cpu().numpy() for t in Wd], [t.cpu().numpy() for t in bd])


def test_nesterov_off_and_custom_coefficients():
    shapes = [(192, 320), (320, 192)]
    W, g, b = _inputs(shapes, 3)
    W_new, b_new = gpu_step(W, g, b, 0.05, 0.9, nesterov=False)
    _check_step(W, g, b, W_new, b_new, lr=0.05, mu=0.9, nesterov=False)
    coeffs = dict(a=2.0, b=-1.5, c=0.5)            # another odd quintic
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95, ns_steps=6, **coeffs)
    _check_step(W, g, b, W_new, b_new, steps=6, **coeffs)


def test_zero_gradient_and_zero_buffer_leave_weights():
    shapes = [(128, 256), (300, 100)]
    W = [np.full(s, 0.25, np.float32) for s in shapes]
    z = [np.zeros(s, np.float32) for s in shapes]
    W_new, b_new = gpu_step(W, z, [x.copy() for x in z], 0.02, 0.95)
    for a, w in zip(W_new, W):
        assert np.array_equal(a, w)
    for x in b_new:
        assert not x.any()


def test_many_matrices_and_classes_split_into_groups():
    # 340 matrices (> 320 per launch) over 18 shapes (> 16 classes per launch)
    shapes = [(64 + 16 * (i % 18), 96 + 40 * (i % 18)) for i in range(340)]
    W, g, b = _inputs(shapes, 4, gscale=0.02)
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    idx = list(range(0, 340, 17)) + [339]
    _check_step([W[i] for i in idx], [g[i] for i in idx], [b[i] for i in idx],
                [W_new[i] for i in idx], [b_new[i] for i in idx])


def test_deterministic_bitwise():
    shapes = [(768, 768), (768, 3072), (3072, 768)]
    W, g, b = _inputs(shapes, 5, gscale=0.02)
    r1 = gpu_step(W, g, b, 0.02, 0.95)
    r2 = gpu_step(W, g, b, 0.02, 0.95)
    for x, y in zip(r1[0] + r1[1], r2[0] + r2[1]):
        assert np.array_equal(x, y)


def test_checkpoint_resume_bitwise():
    w = workloads.get("gpt2_124m")
    idx = [0, 4, 5]                                   # 768x768, 768x3072, 3072x768
    dev = torch.device("cuda:0")
    W0 = workloads.weights(w, indices=idx)
    grads = [workloads.grads(w, s, indices=idx) for s in range(6)]

    def run(W, b, steps):
        Wd = [x.to(dev) for x in W]
        bd = [x.to(dev) for x in b]
        for s in steps:
            muon.step(Wd, [x.to(dev) for x in grads[s]], bd, lr=w.lr, mu=w.mu)
        torch.cuda.synchronize()
        return [x.cpu() for x in Wd], [x.cpu() for x in bd]
    b0 = [torch.zeros_like(x) for x in W0]
    Wa, ba = run(W0, b0, range(6))
    Wm, bm = run(W0, b0, range(3))                    # checkpoint after 3 steps
    Wb, bb = run(Wm, bm, range(3, 6))                 # resume from it
    for x, y in zip(Wa + ba, Wb + bb):
        assert torch.equal(x, y)


def test_prepared_step_matches_step_bitwise():
    shapes = [(256, 768), (768, 256), (130, 250), (64, 2000)]
    W, g, b = _inputs(shapes, seed=31)
    dev = torch.device("cuda:0")
    runs = []
    for prepared in (False, True):
        Wd = [torch.from_numpy(x).to(dev) for x in W]
        bd = [torch.from_numpy(x).to(dev) for x in b]
        gsets = [[torch.from_numpy(x).to(dev) * (1 + k) for x in g] for k in range(3)]
        stepper = muon.PreparedStep(Wd, bd, lr=0.02, mu=0.95) if prepared else None
        for k in range(3):
            if prepared:
                stepper(gsets[k])
            else:
                muon.step(Wd, gsets[k], bd, lr=0.02, mu=0.95)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        runs.append(([x.cpu() for x in Wd], [x.cpu() for x in bd]))
    for a, c in zip(runs[0][0] + runs[0][1], runs[1][0] + runs[1][1]):
        assert torch.equal(a, c)
    with pytest.raises(ValueError, match="shapes differ"):
        stepper([torch.zeros(3, 3, device=dev)] * len(shapes))


def test_host_buffer_entry_point_matches_device_path():
    shapes = [(256, 512), (512, 256)]
    W, g, b = _inputs(shapes, 6)
    W_dev, b_dev = gpu_step(W, g, b, 0.02, 0.95)
    Wh = [torch.as_tensor(x.copy()).pin_memory() for x in W]
    gh = [torch.as_tensor(x.copy()).pin_memory() for x in g]
    bh = [torch.as_tensor(x.copy()).pin_memory() for x in b]
    muon.step_host(Wh, gh, bh, lr=0.02, mu=0.95)
    for x, y in zip(Wh + bh, W_dev + b_dev):
        assert np.array_equal(x.numpy(), y)


def test_host_buffer_entry_point_over_several_chunks_matches_device_path():
    # eight matrices of mixed sizes, more bytes than one 32 MB chunk of the
    # host-buffer pipeline: no path's result depends on which matrices share a
    # launch, so the two entry points agree bitwise
    shapes = [(768, 768), (384, 1024), (1024, 384), (300, 700), (128, 200), (640, 640), (96, 200), (1100, 900)]
    W, g, b = _inputs(shapes, 9)
    W_dev, b_dev = gpu_step(W, g, b, 0.02, 0.95)
    Wh = [torch.as_tensor(x.copy()).pin_memory() for x in W]
    gh = [torch.as_tensor(x.copy()).pin_memory() for x in g]
    bh = [torch.as_tensor(x.copy()).pin_memory() for x in b]
    muon.step_host(Wh, gh, bh, lr=0.02, mu=0.95)
    for x, y in zip(Wh + bh, W_dev + b_dev):
        assert np.array_equal(x.numpy(), y)


@pytest.mark.parametrize("shape,flag", [((384, 384), 1), ((256, 256), 2)], ids=["gemm", "pair"])
def test_bounded_wait_timeout_is_reported_and_context_survives(shape, flag):
    shapes = [shape]
    W, g, b = _inputs(shapes, 7)
    dev = torch.device("cuda:0")
    Wd = [torch.as_tensor(x).to(dev) for x in W]
    gd = [torch.as_tensor(x).to(dev) for x in g]
    bd = [torch.as_tensor(x).to(dev) for x in b]
    muon.debug_set(flag, 20_000_000)                  # next GEMM / pair launch skips a stage; 20 ms bound
    try:
        muon.step(Wd, gd, bd, lr=0.02, mu=0.95)
        assert muon.sync_status() == -5               # MUON_ERR_TIMEOUT
        assert "bounded wait" in muon.last_error()
    finally:
        muon.debug_set(0, 0)
    # the context is still usable and results are right again
    W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
    _check_step(W, g, b, W_new, b_new)


def test_gpt2_124m_ten_steps_against_oracle_subset():
    w = workloads.get("gpt2_124m")
    dev = torch.device("cuda:0")
    Wd = workloads.weights(w, device=dev)
    bd = workloads.zero_bufs(w, device=dev)
    sub = workloads.sample_indices(w, per_shape=2)
    for step in range(w.steps):
        gd = workloads.grads(w, step, device=dev)
        W_pre = [Wd[i].cpu().numpy() for i in sub]
        b_pre = [bd[i].cpu().numpy() for i in sub]
        g_h = [gd[i].cpu().numpy() for i in sub]
        muon.step(Wd, gd, bd, lr=w.lr, mu=w.mu)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0
        for j, i in enumerate(sub):
            W_ref, b_ref, O_ref = muon_oracle.muon_update(W_pre[j], g_h[j], b_pre[j], w.lr, w.mu)
            O = o_from_w(W_pre[j], Wd[i].cpu().numpy(), w.lr)
            check_o(O, O_ref, f"step {step} matrix {i}")
            assert relF(bd[i].cpu().numpy(), b_ref) <= REL_BUF, (step, i)
            if step in (0, w.steps - 1):
                _, G = muon_oracle.momentum_update(g_h[j], b_pre[j], w.mu)
                check_band(O, G)


def test_non_default_eps():
    # eps comparable to ||G||_F changes the scale of X0 and so every
    # singular value the quintic sees; the oracle takes the same eps
    shapes = [(128, 512), (256, 256), (384, 768)]       # single-CTA, CTA-pair and GEMM paths
    W, g, b = _inputs(shapes, 9, gscale=0.01, bscale=0.0)
    for eps in (0.5, 2.0):
        W_new, b_new = gpu_step(W, g, b, 0.02, 0.95, eps=eps)
        _check_step(W, g, b, W_new, b_new, eps=eps)


@pytest.mark.parametrize("poison", [float("nan"), float("inf")], ids=["nan", "inf"])
def test_nan_and_inf_propagate(poison):
    # A non-finite gradient entry makes that matrix's Frobenius norm non-finite,
    # so its whole update is NaN (the arithmetic carries it; nothing checks);
    # its momentum buffer is non-finite exactly where the gradient is, and the
    # other matrices of the same call are unaffected.
    shapes = [(128, 512), (256, 256), (384, 768), (300, 200)]
    W, g, b = _inputs(shapes, 10)
    for bad in range(3):
        g_bad = [x.copy() for x in g]
        g_bad[bad][5, 7] = poison
        W_new, b_new = gpu_step(W, g_bad, b, 0.02, 0.95)
        assert np.isnan(W_new[bad]).all(), f"matrix {bad}: the update is not NaN everywhere"
        assert np.array_equal(~np.isfinite(b_new[bad]), ~np.isfinite(g_bad[bad])), f"buf {bad}"
        ok = [i for i in range(len(shapes)) if i != bad]
        _check_step([W[i] for i in ok], [g[i] for i in ok], [b[i] for i in ok],
                    [W_new[i] for i in ok], [b_new[i] for i in ok])


@pytest.mark.parametrize("ns_steps", [1, 2, 5])
def test_chained_launch_matches_one_launch_per_phase_bitwise(ns_steps):
    # The chained launch computes every tile exactly as the per-phase launches
    # do (same operands, same K order, same epilogue); only the order in which
    # tiles run differs.  So both give bitwise the same weights and buffers.
    shapes = [(768, 768)] * 3 + [(768, 3072), (3072, 768), (640, 1920), (1000, 300), (384, 384), (1024, 1280)]
    W, g, b = _inputs(shapes, 41, gscale=0.02)
    muon.profile_enable(True)
    try:
        muon.profile_read()
        r_chain = gpu_step(W, g, b, 0.02, 0.95, ns_steps=ns_steps)
        kinds = muon.profile_read()
        assert kinds["chain"][1] == 1 and kinds["gram"][1] == 0     # the chained launch ran
        muon.debug_set(4, 0)
        r_phase = gpu_step(W, g, b, 0.02, 0.95, ns_steps=ns_steps)
        kinds = muon.profile_read()
        assert kinds["chain"][1] == 0 and kinds["gram"][1] == ns_steps
    finally:
        muon.debug_set(0, 0)
        muon.profile_enable(False)
    for x, y in zip(r_chain[0] + r_chain[1], r_phase[0] + r_phase[1]):
        assert np.array_equal(x, y)
    _check_step(W, g, b, r_chain[0], r_chain[1], steps=ns_steps)


def test_large_short_sides_take_one_launch_per_phase():
    # short side above 1024: one launch per phase, still within the parity bar
    shapes = [(1600, 1600), (1100, 2000)]
    W, g, b = _inputs(shapes, 43, gscale=0.02)
    muon.profile_enable(True)
    try:
        muon.profile_read()
        W_new, b_new = gpu_step(W, g, b, 0.02, 0.95)
        kinds = muon.profile_read()
    finally:
        muon.profile_enable(False)
    assert kinds["chain"][1] == 0 and kinds["gram"][1] == 5 and kinds["update_apply"][1] == 1
    _check_step(W, g, b, W_new, b_new)
