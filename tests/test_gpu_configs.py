"""GPU parity on every workload at its full size (all matrices run on the GPU
in one call, as the benchmark runs them); a seeded subset of matrices is
checked against the fp64 oracle, and the singular-value band and the momentum
buffer are checked on it as well."""

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon
from muon_newton_schulz_02_b200 import workloads
from oracle import muon_oracle

from gpu_helpers import REL_BUF, check_band, check_o, o_from_w, relF

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _run_and_check(w, steps, subset, band_subset=None, svd_device="cpu"):
    dev = torch.device("cuda:0")
    W = workloads.weights(w, device=dev)
    bufs = workloads.zero_bufs(w, device=dev)
    for step in range(steps):
        g = workloads.grads(w, step, device=dev)
        W_pre = {i: W[i].cpu().numpy() for i in subset}
        b_pre = {i: bufs[i].cpu().numpy() for i in subset}
        g_h = {i: g[i].cpu().numpy() for i in subset}
        muon.step(W, g, bufs, lr=w.lr, mu=w.mu)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        for i in subset:
            W_ref, b_ref, O_ref = muon_oracle.muon_update(W_pre[i], g_h[i], b_pre[i], w.lr, w.mu)
            O = o_from_w(W_pre[i], W[i].cpu().numpy(), w.lr)
            check_o(O, O_ref, f"{w.name} step {step} matrix {i} {w.shapes[i]}")
            assert relF(bufs[i].cpu().numpy(), b_ref) <= REL_BUF, (w.name, step, i)
            if band_subset is not None and i in band_subset and step in (0, steps - 1):
                _, G = muon_oracle.momentum_update(g_h[i], b_pre[i], w.mu)
                check_band(O, G, svd_device=svd_device)
        del g
    del W, bufs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [256, 512, 1024, 2048, 4096])
def test_square_sweep_64_matrices(n):
    w = workloads.get(f"square_n{n}")
    subset = [0, 63]                          # the first and the last matrix of the batch
    _run_and_check(w, 1, subset, band_subset=subset, svd_device="cpu" if n <= 2048 else "cuda:0")


def test_gpt2_xl_five_steps():
    w = workloads.get("gpt2_xl_1p5b")
    subset = [0, 4, 5]                      # 1600x1600, 1600x6400, 6400x1600
    _run_and_check(w, w.steps, subset, band_subset=[0])


def test_illconditioned_lowrank_plus_noise():
    w = workloads.get("illcond_1024x4096")
    subset = [0, 5, 10, 15]
    _run_and_check(w, 1, subset, band_subset=subset)


def test_tall_transpose_path():
    w = workloads.get("tall_8192x1024")
    subset = [0, 15]
    _run_and_check(w, 1, subset, band_subset=[0])
