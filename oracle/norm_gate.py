"""fp64 oracle of the HSTU layer's post-attention step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module; the product path never does.

"Actions Speak Louder than Words" §3 (the HSTU layer, Pointwise
Transformation sub-layer) writes the step after attention as

    Y(X) = Norm(A(X) V(X)) ⊙ U(X)

and names neither the normalisation axis nor its epsilon.  Reading taken:
``Norm`` is a layer normalisation without a learned affine, over the
feature axis of each token, i.e. over the concatenation of all heads'
attention outputs (H·d values per token); the epsilon inside the square root
is a parameter (default 1e-5); the variance is the biased (1/N) one.  ``U`` is
the gate the pointwise projection produced, of the same [T, H·d] shape.

The backward is the exact derivative of the forward with respect to the
attention output and the gate.  Plain numpy in float64, one expression per
step, no blocking or fusion.
"""
from __future__ import annotations

import numpy as np

DEFAULT_EPS = 1e-5


def _rows(a) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    if a.ndim != 2:
        raise ValueError("expected a [T, N] array")
    return a


def norm_gate_fwd(o, u, eps: float = DEFAULT_EPS):
    """Y = LayerNorm(O) ⊙ U per token row.  Returns (y, mean, rstd), each
    float64; ``mean`` and ``rstd`` are [T]."""
    o = _rows(o)
    u = _rows(u)
    if o.shape != u.shape:
        raise ValueError("o and u differ in shape")
    n = o.shape[1]
    mean = o.sum(axis=1) / n
    centred = o - mean[:, None]
    var = (centred * centred).sum(axis=1) / n
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = centred * rstd[:, None]
    return xhat * u, mean, rstd


def norm_gate_bwd(o, u, dy, eps: float = DEFAULT_EPS):
    """Gradients (dO, dU) of sum(dY ⊙ Y) with Y = LayerNorm(O) ⊙ U.

    With x̂ = (o - mean) rstd and g = dY ⊙ U (the gradient reaching x̂):
    dU = x̂ ⊙ dY and dO = rstd (g - mean(g) - x̂ mean(g ⊙ x̂)), the derivative
    of x̂ through the row mean and the row variance."""
    o = _rows(o)
    u = _rows(u)
    dy = _rows(dy)
    if not (o.shape == u.shape == dy.shape):
        raise ValueError("o, u and dy differ in shape")
    n = o.shape[1]
    mean = o.sum(axis=1) / n
    centred = o - mean[:, None]
    var = (centred * centred).sum(axis=1) / n
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = centred * rstd[:, None]
    du = xhat * dy
    g = dy * u
    g_mean = g.sum(axis=1) / n
    gx_mean = (g * xhat).sum(axis=1) / n
    do = rstd[:, None] * (g - g_mean[:, None] - xhat * gx_mean[:, None])
    return do, du
