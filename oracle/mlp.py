"""Unsharded feed-forward sublayer, forward and backward (fp64 NumPy).

Test infrastructure only (see the package docstring).

Definition ("How transformer layers actually decompose"):
    output = GeLU(x W1) W2, x [batch, seq, hidden] flattened to [T, D],
    W1 [D, F], W2 [F, D] (weights are [in, out]).
The pages have no bias; b1 and b2 are added the plain way (b1 before GeLU,
b2 once after the second product), plus an optional residual input r.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .core import gelu, gelu_grad


def mlp_fwd(x, w1, b1, w2, b2, resid: Optional[np.ndarray] = None):
    """Returns (y, a, h): a = x W1 + b1, h = GeLU(a), y = h W2 + b2 (+ r)."""
    a = x @ w1 + b1
    h = gelu(a)
    y = h @ w2 + b2
    if resid is not None:
        y = y + resid
    return y, a, h


def mlp_bwd(x, w1, b1, w2, dy):
    """Vector-Jacobian product of ``mlp_fwd`` for upstream gradient dy.

    Chain rule on y = GeLU(x W1 + b1) W2 + b2:
      dH  = dy W2^T,  dA = dH * GeLU'(A),
      dW2 = H^T dy,   db2 = sum_rows dy,
      dW1 = x^T dA,   db1 = sum_rows dA,
      dx  = dA W1^T.
    The gradient reaching a residual input is dy itself and is not returned.
    Returns a dict with dx, dw1, db1, dw2, db2.
    """
    a = x @ w1 + b1
    h = gelu(a)
    dh = dy @ w2.T
    da = dh * gelu_grad(a)
    return {
        "dx": da @ w1.T,
        "dw1": x.T @ da,
        "db1": da.sum(axis=0),
        "dw2": h.T @ dy,
        "db2": dy.sum(axis=0),
    }
