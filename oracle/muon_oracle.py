"""Oracle for one Muon optimizer step: plain, slow, obviously correct, fp64.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs use it, to check and to time the
CUDA path.  It shares no code with ``muon_newton_schulz_02_b200`` (the CUDA
library and its binding); the only module both sides use is the seeded input
generator ``muon_newton_schulz_02_b200.workloads``, which holds no arithmetic
of the method.

Source of every step (the Modded-NanoGPT news article on jiagew778.com,
"Muon optimizer" section):

* the ``zeroth_power_via_newtonschulz5`` code listing fixes the
  orthogonalisation: normalise by the Frobenius norm plus ``eps=1e-7``, work on
  the transpose when the matrix has more rows than columns, run ``steps=5``
  quintic iterations ``A = X X^T``, ``B = b A + c A A``, ``X = a X + B X`` with
  ``(a, b, c) = (3.4445, -4.7750, 2.0315)``, transpose back;
* the sentence before the listing says the iteration stands in for replacing
  ``G`` by ``U V^T`` from ``G = U S V^T`` (the SVD);
* the "lessons" paragraph says Nesterov momentum is used and the
  orthogonalisation is applied after the momentum.

The article's own formula for the update was an image and did not survive;
this oracle takes the plainest reading that the rest supports:
``buf <- mu*buf + g``; ``G = g + mu*buf`` (Nesterov, using the new buffer);
``W <- W - lr * NS5(G)``.  No shape-dependent learning-rate scale, no weight
decay.

Precision: every step runs in float64 (numpy).  The momentum buffer is state
held in float32 by the caller, so the updated buffer is rounded to float32
when it is stored, and the rest of the step reads that stored value.  The
bf16 casts of the listing are NOT reproduced: the oracle computes the exact
(float64) iteration that the bf16 code approximates.

Pins: every function here is checked in ``tests/test_oracle_pins.py``
against results fixed by the article and by mathematics (the SVD closed form,
exact rational arithmetic on diagonal inputs, invariances, the limiting band
quoted in the lessons paragraph, the momentum closed form).
"""

from __future__ import annotations

import numpy as np

# Quintic coefficients, step count and epsilon: the defaults of the
# zeroth_power_via_newtonschulz5 listing ("Muon optimizer" section).
NS_A = 3.4445
NS_B = -4.7750
NS_C = 2.0315
NS_STEPS = 5
NS_EPS = 1e-7


def quintic(x, a=NS_A, b=NS_B, c=NS_C):
    """The scalar map one NS5 iteration applies to each singular value:
    p(x) = a x + b x^3 + c x^5 (follows from A = X X^T, B = b A + c A A,
    X = a X + B X applied to X = U diag(x) V^T)."""
    return a * x + b * x**3 + c * x**5


def newton_schulz5(G, steps=NS_STEPS, eps=NS_EPS, a=NS_A, b=NS_B, c=NS_C):
    """NewtonSchulz5(G): the quintic Newton-Schulz orthogonalisation of one
    2-D matrix, in float64 (the article's definition sentence names it; its
    code listing, zeroth_power_via_newtonschulz5, fixes the steps).

    The iteration works on the wide orientation (rows <= cols) of G scaled to
    unit Frobenius norm (plus eps); each of the ``steps`` rounds forms the
    Gram matrix A of the iterate, the polynomial B = b A + c A^2 in it, and
    the next iterate a X + B X.  The result is brought back to G's
    orientation.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("NS5 is defined for 2-D matrices only")
    X = G / (np.linalg.norm(G) + eps)          # Frobenius norm of the whole matrix
    transposed = G.shape[0] > G.shape[1]
    if transposed:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    if transposed:
        X = X.T
    return X


def momentum_update(g, buf, mu, nesterov=True):
    """Momentum step of the Muon update ("lessons" paragraph: Nesterov
    momentum, orthogonalisation after the momentum).

    Returns (new_buf as float32, G as float64) with
    new_buf = mu*buf + g and G = g + mu*new_buf (Nesterov) or G = new_buf.
    ``mu`` is taken at float32 precision, as the caller's state is float32.
    """
    mu64 = float(np.float32(mu))
    g64 = np.asarray(g, dtype=np.float32).astype(np.float64)
    buf64 = np.asarray(buf, dtype=np.float32).astype(np.float64)
    new_buf = (mu64 * buf64 + g64).astype(np.float32)
    if nesterov:
        G = g64 + mu64 * new_buf.astype(np.float64)
    else:
        G = new_buf.astype(np.float64)
    return new_buf, G


def muon_update(W, g, buf, lr, mu, steps=NS_STEPS, nesterov=True,
                eps=NS_EPS, a=NS_A, b=NS_B, c=NS_C):
    """One Muon step on one weight matrix.

    Returns (W_new float32, buf_new float32, O float64) where O is the
    orthogonalised update and W_new = W - lr*O (computed in float64 from the
    float32 W, then stored as float32).
    """
    new_buf, G = momentum_update(g, buf, mu, nesterov)
    O = newton_schulz5(G, steps=steps, eps=eps, a=a, b=b, c=c)
    lr64 = float(np.float32(lr))
    W_new = (np.asarray(W, dtype=np.float32).astype(np.float64) - lr64 * O).astype(np.float32)
    return W_new, new_buf, O

