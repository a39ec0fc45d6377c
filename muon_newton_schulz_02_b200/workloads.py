"""Seeded synthetic workloads for the Muon step.

This module only draws random inputs; it holds none of the Muon arithmetic.
It is the one module that both the CUDA path's tests/bench and the CPU
oracle's tests use, so that both sides see the same arrays.

Shapes follow the GPT-2 layer sets of the Modded-NanoGPT speedrun context
(124M: 12 layers of q,k,v,o 768x768 plus fc 768x3072 and proj 3072x768;
1.5B: 48 layers of 1600x1600 x4, 1600x6400, 6400x1600), a square sweep, and an
ill-conditioned / tall stress set.

Every matrix is drawn from its own generator seeded by
``(base_seed + step) * 4096 + index`` (gradients) or
``(base_seed + 777) * 4096 + index`` (weights), so any one matrix can be
regenerated alone.  Draws on the CPU use torch's CPU generator; draws on a CUDA
device use that device's generator, which yields different (but equally
seeded and deterministic) values; a test always hands the very same host
copy to both sides.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    shapes: tuple            # ((rows, cols), ...)
    grad_std: float          # std of the N(0, std) gradient entries (0 => special)
    base_seed: int
    steps: int               # consecutive Muon steps the workload runs
    mu: float = 0.95
    lr: float = 0.02
    weight_std: float = 0.02
    kind: str = "gaussian"   # "gaussian" | "lowrank_plus_noise"
    extra: dict = field(default_factory=dict)

    @property
    def n_matrices(self) -> int:
        return len(self.shapes)

    @property
    def n_elements(self) -> int:
        return sum(r * c for r, c in self.shapes)


def _gpt2_shapes(layers: int, d: int) -> tuple:
    per_layer = [(d, d)] * 4 + [(d, 4 * d), (4 * d, d)]
    return tuple(per_layer * layers)


WORKLOADS = {
    "single_128x512": Workload("single_128x512", ((128, 512),), 1.0, 1000, 1),
    "gpt2_124m": Workload("gpt2_124m", _gpt2_shapes(12, 768), 0.02, 2000, 10),
    "gpt2_xl_1p5b": Workload("gpt2_xl_1p5b", _gpt2_shapes(48, 1600), 0.02, 4000, 5),
    "illcond_1024x4096": Workload(
        "illcond_1024x4096", ((1024, 4096),) * 16, 0.0, 5000, 1,
        kind="lowrank_plus_noise",
        extra={"rank": 64, "log_s_min": math.log(1e-6), "log_s_max": 0.0, "noise_std": 1e-4}),
    "tall_8192x1024": Workload("tall_8192x1024", ((8192, 1024),) * 16, 1.0, 5001, 1),
}
for _n in (256, 512, 1024, 2048, 4096):
    WORKLOADS[f"square_n{_n}"] = Workload(f"square_n{_n}", ((_n, _n),) * 64, 1.0, 3000 + _n, 1)


def get(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _lowrank_plus_noise(rows, cols, ex, g, device):
    """U diag(s) V^T + noise with Haar-distributed orthonormal U, V (QR of a
    Gaussian, columns sign-fixed by diag(R)) and log-uniform s."""
    r = ex["rank"]
    qa, ra = torch.linalg.qr(torch.randn(rows, r, generator=g, device=device, dtype=torch.float64))
    qa = qa * torch.sign(torch.diagonal(ra)).unsqueeze(0)
    qb, rb = torch.linalg.qr(torch.randn(cols, r, generator=g, device=device, dtype=torch.float64))
    qb = qb * torch.sign(torch.diagonal(rb)).unsqueeze(0)
    u = torch.rand(r, generator=g, device=device, dtype=torch.float64)
    s = torch.exp(ex["log_s_min"] + (ex["log_s_max"] - ex["log_s_min"]) * u)
    noise = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float64) * ex["noise_std"]
    return ((qa * s.unsqueeze(0)) @ qb.T + noise).to(torch.float32)


def grad(w: Workload, step: int, index: int, device="cpu") -> torch.Tensor:
    """Gradient matrix ``index`` of step ``step`` (float32, contiguous)."""
    rows, cols = w.shapes[index]
    g = _gen(device, (w.base_seed + step) * 4096 + index)
    if w.kind == "lowrank_plus_noise":
        return _lowrank_plus_noise(rows, cols, w.extra, g, device)
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * w.grad_std


def weight(w: Workload, index: int, device="cpu") -> torch.Tensor:
    rows, cols = w.shapes[index]
    g = _gen(device, (w.base_seed + 777) * 4096 + index)
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * w.weight_std


def grads(w: Workload, step: int, device="cpu", indices=None):
    idx = range(w.n_matrices) if indices is None else indices
    return [grad(w, step, i, device) for i in idx]


def weights(w: Workload, device="cpu", indices=None):
    idx = range(w.n_matrices) if indices is None else indices
    return [weight(w, i, device) for i in idx]


def zero_bufs(w: Workload, device="cpu", indices=None):
    idx = range(w.n_matrices) if indices is None else indices
    return [torch.zeros(w.shapes[i], device=device, dtype=torch.float32) for i in idx]


def sample_indices(w: Workload, per_shape: int = 2):
    """A fixed subset: the first ``per_shape`` matrices of every distinct shape."""
    seen, out = {}, []
    for i, s in enumerate(w.shapes):
        if seen.get(s, 0) < per_shape:
            seen[s] = seen.get(s, 0) + 1
            out.append(i)
    return out
