"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the CPU oracle on the same host arrays."""

import numpy as np
import torch

import muon_newton_schulz_02_b200 as muon
from oracle import muon_oracle

# Parity bar: relative Frobenius error of the orthogonalised update against
# the fp64 oracle; fp32 momentum buffer; singular-value band of the output.
REL_O = 3e-2
REL_BUF = 1e-6
BAND_LO, BAND_HI = 0.6, 1.21
X_THRESHOLD = 1.302e-3      # p^5(x) >= 0.6 exactly for x above this


def relF(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


# Blockwise bar: every BLOCK x BLOCK block of O must match the oracle's block
# to REL_BLOCK of that block's norm, plus a floor of FLOOR_BLOCK times the
# matrix's root-mean-square block norm (so that blocks the oracle leaves near
# zero, as in a low-rank input, are not judged on their own tiny norm).  A
# wrong or stale tile is a large error in its own blocks even where it is a
# small part of the whole matrix's Frobenius norm.
BLOCK = 128
REL_BLOCK = 6e-2
FLOOR_BLOCK = 1e-3


def block_errors(O, ref, bs=BLOCK):
    """Worst ratio err_B / (REL_BLOCK*||ref_B|| + floor) over all blocks (<= 1
    passes), and the worst block's (row, col) origin."""
    O = np.asarray(O, np.float64)
    ref = np.asarray(ref, np.float64)
    m, n = ref.shape
    nb = ((m + bs - 1) // bs) * ((n + bs - 1) // bs)
    floor = FLOOR_BLOCK * np.linalg.norm(ref) / np.sqrt(nb)
    worst, where = 0.0, (0, 0)
    for i in range(0, m, bs):
        for j in range(0, n, bs):
            rb = ref[i:i + bs, j:j + bs]
            eb = np.linalg.norm(O[i:i + bs, j:j + bs] - rb)
            ratio = eb / (REL_BLOCK * np.linalg.norm(rb) + floor) if eb > 0 else 0.0
            if ratio > worst:
                worst, where = ratio, (i, j)
    return worst, where


def check_o(O, ref, what=""):
    """The parity bar on one orthogonalised update: relF <= REL_O and every
    block within the blockwise bar.  Returns (relF, worst block ratio)."""
    err = relF(O, ref)
    assert err <= REL_O, f"{what}: relF(O) = {err:.3e} > {REL_O}"
    worst, where = block_errors(O, ref)
    assert worst <= 1.0, f"{what}: block at {where} off by {worst:.2f} x the blockwise bar (relF {err:.3e})"
    return err, worst


def o_from_w(W_old, W_new, lr):
    return (np.asarray(W_old, np.float64) - np.asarray(W_new, np.float64)) / float(np.float32(lr))


def check_band(O, G, svd_device="cpu"):
    """Every singular value of O <= BAND_HI; no more values below BAND_LO than
    normalised input singular values below X_THRESHOLD.  An output singular
    value counts as below BAND_LO only if it is below it by more than the
    parity tolerance REL_O: an input just above the threshold maps to just
    above 0.6 in exact arithmetic, and the bf16 iteration may move it by that
    much."""
    if svd_device == "cpu":
        so = np.linalg.svd(np.asarray(O, np.float64), compute_uv=False)
        sg = np.linalg.svd(np.asarray(G, np.float64), compute_uv=False)
    else:
        so = torch.linalg.svdvals(torch.as_tensor(O, device=svd_device, dtype=torch.float64)).cpu().numpy()
        sg = torch.linalg.svdvals(torch.as_tensor(G, device=svd_device, dtype=torch.float64)).cpu().numpy()
    x = sg / (np.sqrt((sg ** 2).sum()) + 1e-7)
    n_small_in = int((x < X_THRESHOLD).sum())
    n_low_out = int((so < BAND_LO * (1 - REL_O)).sum())
    assert so.max() <= BAND_HI, f"max singular value {so.max():.5f} above {BAND_HI}"
    assert n_low_out <= n_small_in, f"{n_low_out} singular values < {BAND_LO}, only {n_small_in} inputs below threshold"
    return so


def gpu_step(W, g, buf, lr, mu, ns_steps=5, **kw):
    """Copies host fp32 arrays to cuda:0, runs muon.step, returns host results."""
    dev = torch.device("cuda:0")
    Wd = [torch.as_tensor(w).to(dev) for w in W]
    gd = [torch.as_tensor(x).to(dev) for x in g]
    bd = [torch.as_tensor(b).to(dev) for b in buf]
    muon.step(Wd, gd, bd, lr=lr, mu=mu, ns_steps=ns_steps, **kw)
    torch.cuda.synchronize()
    assert muon.sync_status() == 0, muon.last_error()
    return [w.cpu().numpy() for w in Wd], [b.cpu().numpy() for b in bd]
