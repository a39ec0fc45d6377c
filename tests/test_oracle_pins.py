"""Pins for the CPU oracle: results fixed by the article and by mathematics,
independent of the oracle's own code path.

* SVD closed form (the article: NS5 stands in for G -> U V^T): for
  G = U S V^T, NS5 returns U p^5(S/(||G||+eps)) V^T with p(x)=ax+bx^3+cx^5,
  checked with LAPACK's SVD and with a one-sided Jacobi SVD written here.
* Diagonal inputs map entrywise; checked in exact rational arithmetic.
* Invariances: transpose, sign, orthogonal factors, scale, zero padding, rank.
* The limiting band of repeated application quoted in the lessons paragraph.
* Momentum closed form for a constant gradient.
* A few planted mistakes in a copy of the oracle, each caught by a pin above.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import muon_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ns5_constants.json")


def _p5_scalar(x, steps=5):
    for _ in range(steps):
        x = orc.NS_A * x + orc.NS_B * x**3 + orc.NS_C * x**5
    return x


def _closed_form_lapack(G, steps=5, eps=orc.NS_EPS):
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    x = s / (np.sqrt((s**2).sum()) + eps)        # ||G||_F from the spectrum
    return (U * _p5_scalar(x, steps)) @ Vt


def _jacobi_svd(A, sweeps=60, tol=1e-15):
    """One-sided (Hestenes) Jacobi SVD, thin form, written out here so that
    the pin does not rest on LAPACK.  Returns U, s, V with A = U diag(s) V^T."""
    A = np.array(A, dtype=np.float64)
    flip = A.shape[0] < A.shape[1]
    if flip:
        A = A.T
    m, n = A.shape
    V = np.eye(n)
    for _ in range(sweeps):
        off = 0.0
        for i in range(n - 1):
            for j in range(i + 1, n):
                ai, aj = A[:, i], A[:, j]
                alpha, beta, gamma = ai @ ai, aj @ aj, ai @ aj
                if abs(gamma) <= tol * np.sqrt(alpha * beta) or gamma == 0.0:
                    continue
                off = max(off, abs(gamma) / np.sqrt(alpha * beta))
                zeta = (beta - alpha) / (2.0 * gamma)
                t = np.sign(zeta) / (abs(zeta) + np.sqrt(1.0 + zeta * zeta)) if zeta != 0 else 1.0
                cs = 1.0 / np.sqrt(1.0 + t * t)
                sn = cs * t
                Ai, Aj = A[:, i].copy(), A[:, j].copy()
                A[:, i], A[:, j] = cs * Ai - sn * Aj, sn * Ai + cs * Aj
                Vi, Vj = V[:, i].copy(), V[:, j].copy()
                V[:, i], V[:, j] = cs * Vi - sn * Vj, sn * Vi + cs * Vj
        if off < tol:
            break
    s = np.sqrt((A * A).sum(axis=0))
    U = A / np.where(s > 0, s, 1.0)
    if flip:
        return V, s, U
    return U, s, V


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(np.asarray(b)))


# ------------------------------------------------------------- constants ---

def test_constants_match_listing():
    gold = json.load(open(GOLDEN))
    assert orc.NS_A == gold["coefficients"]["a"]
    assert orc.NS_B == gold["coefficients"]["b"]
    assert orc.NS_C == gold["coefficients"]["c"]
    assert orc.NS_STEPS == gold["steps"]["value"]
    assert orc.NS_EPS == gold["eps"]["value"]


def test_quintic_scalar_facts():
    # p(1) = a + b + c, p'(0) = a: the listing's coefficients, maximal slope at 0.
    assert abs(orc.quintic(1.0) - 0.701) < 1e-12
    h = 1e-7
    assert abs((orc.quintic(h) - orc.quintic(-h)) / (2 * h) - orc.NS_A) < 1e-9
    assert orc.quintic(0.0) == 0.0                       # odd polynomial: rank preserved


def test_repeated_quintic_band_matches_lessons_paragraph():
    gold = json.load(open(GOLDEN))["limit_band"]
    x = np.linspace(1e-3, 1.0, 20001)
    for _ in range(200):
        x = orc.quintic(x)
    # "converges to about 0.68 .. 1.13": both ends reached to two decimals.
    assert abs(x.min() - gold["low"]) < 5e-3
    assert abs(x.max() - gold["high"]) < 5e-3


def test_repeated_ns_on_matrix_lands_in_band():
    rng = np.random.default_rng(7)
    G = rng.standard_normal((24, 40))
    O = orc.newton_schulz5(G, steps=60)
    s = np.linalg.svd(O, compute_uv=False)
    assert s.min() > 0.675 and s.max() < 1.135


# ------------------------------------------------------- SVD closed form ---

@pytest.mark.parametrize("shape", [(4, 3), (3, 5), (16, 16), (64, 40), (40, 64), (128, 512), (300, 96)])
def test_svd_closed_form_lapack(shape):
    rng = np.random.default_rng(hash(shape) % 2**32)
    G = rng.standard_normal(shape) * 0.3
    O = orc.newton_schulz5(G)
    assert O.shape == G.shape
    assert _rel(O, _closed_form_lapack(G)) < 1e-12


@pytest.mark.parametrize("shape", [(5, 3), (3, 5), (8, 8), (12, 7), (6, 16)])
def test_svd_closed_form_jacobi(shape):
    rng = np.random.default_rng(11 + shape[0] * 31 + shape[1])
    G = rng.standard_normal(shape)
    U, s, V = _jacobi_svd(G)
    assert _rel((U * s) @ V.T, G) < 1e-13                  # the Jacobi SVD itself
    x = s / (np.linalg.norm(s) + orc.NS_EPS)
    expect = (U * _p5_scalar(x)) @ V.T
    assert _rel(orc.newton_schulz5(G), expect) < 1e-12


@pytest.mark.parametrize("steps", [0, 1, 2, 7])
def test_svd_closed_form_other_step_counts(steps):
    rng = np.random.default_rng(100 + steps)
    G = rng.standard_normal((20, 33))
    assert _rel(orc.newton_schulz5(G, steps=steps),
                _closed_form_lapack(G, steps=steps)) < 1e-12


def test_zero_steps_is_normalisation():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((9, 4))
    O = orc.newton_schulz5(G, steps=0)
    assert np.allclose(O, G / (np.linalg.norm(G) + 1e-7), rtol=0, atol=1e-15)


# --------------------------------------------- diagonal, exact rationals ---

def _exact_p5(d, norm, eps, steps=5):
    a, b, c = Fraction(orc.NS_A), Fraction(orc.NS_B), Fraction(orc.NS_C)
    x = Fraction(d) / (Fraction(norm) + Fraction(eps))
    for _ in range(steps):
        x = a * x + b * x**3 + c * x**5
    return x


@pytest.mark.parametrize("shape", [(4, 6), (6, 4), (4, 4)])
def test_diagonal_input_exact_rational(shape):
    d = [1.0, -2.0, 2.0, 4.0]                 # ||d|| = 5 exactly
    G = np.zeros(shape)
    for i, v in enumerate(d):
        G[i, i] = v
    O = orc.newton_schulz5(G)
    mask = np.zeros(shape, dtype=bool)
    for i, v in enumerate(d):
        mask[i, i] = True
        exact = float(_exact_p5(v, 5.0, orc.NS_EPS))
        assert abs(O[i, i] - exact) <= 1e-13 * abs(exact)
        assert np.sign(O[i, i]) == np.sign(v)            # p is odd
    assert np.all(O[~mask] == 0.0)


# ------------------------------------------------------------ invariances ---

def test_transpose_symmetry():
    rng = np.random.default_rng(5)
    G = rng.standard_normal((30, 70))
    assert np.array_equal(orc.newton_schulz5(G.T),
                          orc.newton_schulz5(G).T)


def test_sign_and_orthogonal_invariance():
    rng = np.random.default_rng(6)
    G = rng.standard_normal((20, 35))
    O = orc.newton_schulz5(G)
    assert np.array_equal(orc.newton_schulz5(-G), -O)
    Q, _ = np.linalg.qr(rng.standard_normal((20, 20)))
    R, _ = np.linalg.qr(rng.standard_normal((35, 35)))
    assert _rel(orc.newton_schulz5(Q @ G @ R), Q @ O @ R) < 1e-12


@pytest.mark.parametrize("scale", [1e-3, 1e3])
def test_scale_invariance(scale):
    rng = np.random.default_rng(8)
    G = rng.standard_normal((16, 48))
    a = orc.newton_schulz5(G * scale, eps=0.0)
    b = orc.newton_schulz5(G, eps=0.0)
    assert _rel(a, b) < 1e-12
    # with the default eps the only difference is eps against the norm
    c = orc.newton_schulz5(G * scale)
    assert _rel(c, b) < 1e-5


@pytest.mark.parametrize("pad", [(0, 5), (5, 0), (7, 9), (40, 0)])
def test_zero_padding_leaves_block_unchanged(pad):
    rng = np.random.default_rng(9)
    G = rng.standard_normal((12, 20))
    P = np.zeros((12 + pad[0], 20 + pad[1]))
    P[:12, :20] = G
    O = orc.newton_schulz5(P)
    assert _rel(O[:12, :20], orc.newton_schulz5(G)) < 1e-12
    assert np.all(O[12:, :] == 0.0) and np.all(O[:, 20:] == 0.0)


def test_rank_preserved():
    rng = np.random.default_rng(10)
    G = rng.standard_normal((30, 3)) @ rng.standard_normal((3, 50))
    s = np.linalg.svd(orc.newton_schulz5(G), compute_uv=False)
    assert np.all(s[:3] > 0.5) and np.all(s[3:] < 1e-10)


# --------------------------------------------------------------- momentum ---

@pytest.mark.parametrize("mu", [0.95, 0.5])
def test_momentum_closed_form_constant_gradient(mu):
    rng = np.random.default_rng(12)
    g = rng.standard_normal((6, 5)).astype(np.float32)
    buf = np.zeros_like(g)
    T = 25
    for _ in range(T):
        buf, G = orc.momentum_update(g, buf, mu, nesterov=True)
    mu32 = float(np.float32(mu))
    expect = g.astype(np.float64) * (1 - mu32**T) / (1 - mu32)
    assert _rel(buf, expect) < 1e-6
    assert _rel(G, g + mu32 * expect) < 1e-6


def test_momentum_variants():
    rng = np.random.default_rng(13)
    g = rng.standard_normal((4, 7)).astype(np.float32)
    buf = rng.standard_normal((4, 7)).astype(np.float32)
    nb, G = orc.momentum_update(g, buf, 0.9, nesterov=False)
    assert np.array_equal(G, nb.astype(np.float64))
    nb0, G0 = orc.momentum_update(g, np.zeros_like(g), 0.0)
    assert np.array_equal(G0, g.astype(np.float64)) and np.array_equal(nb0, g)


def test_muon_update_mu_zero_is_plain_ns5_and_applies_lr():
    rng = np.random.default_rng(14)
    W = (rng.standard_normal((10, 24)) * 0.02).astype(np.float32)
    g = rng.standard_normal((10, 24)).astype(np.float32)
    W_new, b_new, O = orc.muon_update(W, g, np.zeros_like(g), lr=0.02, mu=0.0)
    assert _rel(O, orc.newton_schulz5(g.astype(np.float64))) < 1e-15
    lr = float(np.float32(0.02))
    assert np.array_equal(W_new, (W.astype(np.float64) - lr * O).astype(np.float32))
    assert np.array_equal(b_new, g)


@pytest.mark.parametrize("shape", [(12, 30), (30, 12), (9, 9)])
@pytest.mark.parametrize("lr", [1.0, 0.02])
def test_muon_update_apply_matches_svd_closed_form(shape, lr):
    # With mu = 0 the momentum step passes g through, and with W = 0 the new
    # weights are -lr times the orthogonalised gradient: W_new must equal
    # -lr * U p^5(S/(||g||+eps)) V^T, the replacement of G by (a smoothed)
    # U V^T that the article's definition sentence states, from LAPACK and
    # from the Jacobi SVD written here.
    rng = np.random.default_rng(20 + shape[0] + 7 * shape[1])
    g = rng.standard_normal(shape).astype(np.float32)
    W0 = np.zeros(shape, dtype=np.float32)
    W_new, b_new, O = orc.muon_update(W0, g, np.zeros_like(g), lr=lr, mu=0.0)
    g64 = g.astype(np.float64)
    lr64 = float(np.float32(lr))
    U, s, V = _jacobi_svd(g64)
    x = s / (np.linalg.norm(s) + orc.NS_EPS)
    for ref in (-lr64 * _closed_form_lapack(g64), -lr64 * (U * _p5_scalar(x)) @ V.T):
        # W_new is stored in float32: one rounding of each entry
        assert np.max(np.abs(W_new - ref)) <= 2.0 ** -23 * np.max(np.abs(ref)) * 2
        assert _rel(W_new, ref) < 1e-6
    assert np.array_equal(b_new, g)


def test_muon_update_apply_adds_to_existing_weights():
    # W_new - W is the same -lr * O for any W (the update is additive): two
    # starting points that differ by a constant matrix end up differing by it.
    rng = np.random.default_rng(31)
    g = rng.standard_normal((8, 20)).astype(np.float32)
    W1 = np.zeros((8, 20), dtype=np.float32)
    W2 = np.full((8, 20), 0.5, dtype=np.float32)       # 0.5 - lr*O stays exact enough in fp32
    a1, _, _ = orc.muon_update(W1, g, np.zeros_like(g), lr=0.25, mu=0.0)
    a2, _, _ = orc.muon_update(W2, g, np.zeros_like(g), lr=0.25, mu=0.0)
    assert np.max(np.abs((a2.astype(np.float64) - 0.5) - a1)) < 1e-6


def test_zero_gradient_leaves_weights():
    W = np.full((3, 8), 0.5, dtype=np.float32)
    g = np.zeros((3, 8), dtype=np.float32)
    W_new, b_new, O = orc.muon_update(W, g, np.zeros_like(g), 0.02, 0.95)
    assert np.all(O == 0) and np.array_equal(W_new, W) and np.all(b_new == 0)


# ------------------------------------------------------ planted mistakes ---
# Copies of the oracle with one deliberate error each; every one must fail a
# pin above (here: the SVD closed form on a non-square input).

def _ns5_variant(G, mistake, steps=5, eps=1e-7):
    a, b, c = orc.NS_A, orc.NS_B, orc.NS_C
    if mistake == "swap_bc":
        b, c = c, b
    norm = np.linalg.norm(G)
    X = G / ((norm * norm if mistake == "norm_squared" else norm) + eps)
    t = G.shape[0] > G.shape[1]
    if t:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = (a * X + B @ X) if mistake != "drop_aX" else (B @ X)
        if mistake == "transpose_inside_loop":
            X = X.T
    if t and mistake != "no_transpose_back":
        X = X.T
    return X


@pytest.mark.parametrize("mistake", ["swap_bc", "drop_aX", "no_transpose_back", "norm_squared",
                                     "transpose_inside_loop"])
def test_planted_mistakes_are_caught(mistake):
    rng = np.random.default_rng(15)
    # tall input exercises the transpose; a square one shows a stray transpose
    shape = (32, 32) if mistake == "transpose_inside_loop" else (40, 24)
    G = rng.standard_normal(shape)
    try:
        O = _ns5_variant(G, mistake)
        err = _rel(O, _closed_form_lapack(G)) if O.shape == G.shape else np.inf
    except ValueError:
        err = np.inf
    assert err > 1e-3


# Planted mistakes in the apply (copies of muon_update with one error each):
# each must fail the SVD closed-form pin of the apply above.
def _update_variant(W, g, lr, mistake):
    O = orc.newton_schulz5(np.asarray(g, np.float64))
    lr64 = float(np.float32(lr))
    W64 = np.asarray(W, np.float64)
    if mistake == "apply_sign":
        return (W64 + lr64 * O).astype(np.float32)
    if mistake == "lr_applied_twice":
        return (W64 - lr64 * lr64 * O).astype(np.float32)
    if mistake == "apply_transposed":
        return (W64 - lr64 * O.T).astype(np.float32) if O.shape[0] == O.shape[1] else None
    raise ValueError(mistake)


@pytest.mark.parametrize("mistake", ["apply_sign", "lr_applied_twice", "apply_transposed"])
def test_planted_apply_mistakes_are_caught(mistake):
    rng = np.random.default_rng(16)
    shape = (10, 10) if mistake == "apply_transposed" else (10, 26)
    g = rng.standard_normal(shape).astype(np.float32)
    lr = 0.02
    W_bad = _update_variant(np.zeros(shape, np.float32), g, lr, mistake)
    ref = -float(np.float32(lr)) * _closed_form_lapack(g.astype(np.float64))
    assert _rel(W_bad, ref) > 1e-3
    # and the oracle itself passes the same check
    W_ok, _, _ = orc.muon_update(np.zeros(shape, np.float32), g, np.zeros_like(g), lr=lr, mu=0.0)
    assert _rel(W_ok, ref) < 1e-6
