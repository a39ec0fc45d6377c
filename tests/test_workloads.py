"""The seeded synthetic workloads: shapes and counts as documented, per-matrix
regeneration, determinism, the stated distributions, and the spectrum of the
ill-conditioned set.  CPU only."""

import math
from collections import Counter

import numpy as np
import pytest
import torch

from muon_newton_schulz_02_b200 import workloads


def test_shapes_and_counts():
    assert workloads.get("single_128x512").shapes == ((128, 512),)
    gpt2 = Counter(workloads.get("gpt2_124m").shapes)
    assert gpt2 == {(768, 768): 48, (768, 3072): 12, (3072, 768): 12}
    xl = Counter(workloads.get("gpt2_xl_1p5b").shapes)
    assert xl == {(1600, 1600): 192, (1600, 6400): 48, (6400, 1600): 48}
    for n in (256, 512, 1024, 2048, 4096):
        assert workloads.get(f"square_n{n}").shapes == ((n, n),) * 64
    assert workloads.get("illcond_1024x4096").shapes == ((1024, 4096),) * 16
    assert workloads.get("tall_8192x1024").shapes == ((8192, 1024),) * 16
    assert workloads.get("gpt2_124m").n_elements == 48 * 768 * 768 + 24 * 768 * 3072
    with pytest.raises(KeyError):
        workloads.get("no_such_workload")


def test_matrices_regenerate_alone_and_deterministically():
    w = workloads.get("gpt2_124m")
    full = workloads.grads(w, 3, indices=range(8))
    for i in range(8):
        assert torch.equal(full[i], workloads.grad(w, 3, i))
    assert torch.equal(workloads.weight(w, 5), workloads.weights(w)[5])
    assert not torch.equal(workloads.grad(w, 3, 0), workloads.grad(w, 4, 0))     # steps differ
    assert not torch.equal(workloads.grad(w, 3, 0), workloads.grad(w, 3, 1)[:768, :768])
    assert not torch.equal(workloads.weight(w, 0), workloads.grad(w, 0, 0))
    z = workloads.zero_bufs(w, indices=[4])[0]
    assert z.shape == (768, 3072) and z.dtype == torch.float32 and not z.any()


@pytest.mark.parametrize("name,std", [("gpt2_124m", 0.02), ("single_128x512", 1.0), ("square_n512", 1.0)])
def test_gaussian_gradients_and_weights_have_the_stated_std(name, std):
    w = workloads.get(name)
    g = workloads.grad(w, 0, 0).double()
    assert g.dtype == torch.float64 and g.is_contiguous()
    assert abs(float(g.mean())) < 5 * std / math.sqrt(g.numel())
    assert abs(float(g.std()) / std - 1) < 0.02
    W = workloads.weight(w, 0).double()
    assert abs(float(W.std()) / w.weight_std - 1) < 0.02


def test_illconditioned_spectrum_is_lowrank_log_uniform_plus_noise():
    w = workloads.get("illcond_1024x4096")
    ex = w.extra
    G = workloads.grad(w, 0, 0).double().numpy()
    s = np.linalg.svd(G, compute_uv=False)
    m, n = G.shape
    noise_edge = ex["noise_std"] * (math.sqrt(m) + math.sqrt(n))     # largest singular value of the noise
    assert s[0] <= math.exp(ex["log_s_max"]) + 2 * noise_edge        # the signal's are <= 1
    assert 0.8 * noise_edge < s[ex["rank"]] < 1.2 * noise_edge       # beyond the rank: noise only
    assert (s > 0.05).sum() <= ex["rank"]
    # the signal's singular values above the noise spread over decades (log-uniform)
    big = s[s > 5 * noise_edge]
    assert len(big) >= 10 and big.max() / big.min() > 10


def test_sample_indices_take_the_first_of_every_shape():
    w = workloads.get("gpt2_124m")
    idx = workloads.sample_indices(w, per_shape=2)
    assert idx == [0, 1, 4, 5, 10, 11]
    assert Counter(w.shapes[i] for i in idx) == {(768, 768): 2, (768, 3072): 2, (3072, 768): 2}


def test_module_holds_no_method_arithmetic():
    import ast
    tree = ast.parse(open(workloads.__file__).read())
    imported = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            imported |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom):
            imported.add((node.module or "").split(".")[0])
    assert imported <= {"__future__", "math", "dataclasses", "torch"}      # neither oracle nor library
    constants = {n.value for n in ast.walk(tree) if isinstance(n, ast.Constant) and isinstance(n.value, float)}
    assert not constants & {3.4445, -4.775, 4.775, 2.0315}                 # no quintic coefficients
