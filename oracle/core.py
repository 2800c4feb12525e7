"""Elementwise and row-wise building blocks of the oracle (fp64 NumPy).

Test infrastructure only (see the package docstring).
"""
from __future__ import annotations

import math

import numpy as np

# tanh form of GeLU (Hendrycks & Gimpel 2016).  The pages name only "GeLU"
# ("How transformer layers actually decompose": output = GeLU(xW1) W2); the
# MLP workload names the tanh form and nothing contradicts it, so every
# workload uses it.
GELU_C = math.sqrt(2.0 / math.pi)
GELU_A = 0.044715


def gelu(a: np.ndarray) -> np.ndarray:
    """0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3)))."""
    return 0.5 * a * (1.0 + np.tanh(GELU_C * (a + GELU_A * a ** 3)))


def gelu_grad(a: np.ndarray) -> np.ndarray:
    """d/da of ``gelu``, by the product and chain rules.

    With u = c (a + k a^3): d/da [0.5 a (1 + tanh u)]
      = 0.5 (1 + tanh u) + 0.5 a (1 - tanh^2 u) c (1 + 3 k a^2).
    """
    u = GELU_C * (a + GELU_A * a ** 3)
    th = np.tanh(u)
    return 0.5 * (1.0 + th) + 0.5 * a * (1.0 - th * th) * GELU_C * (1.0 + 3.0 * GELU_A * a * a)


def layernorm_fwd(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = 1e-5):
    """LayerNorm over the last axis, biased variance (divide by D).

    Pre-LN placement ("The layernorm placement the paper flags as critical").
    The pages fix neither eps nor the variance estimator; eps = 1e-5 and the
    biased variance are the plain reading.
    Returns (y, mean, rstd) with y = (x - mean) * rstd * gamma + beta.
    """
    mean = x.mean(axis=-1)
    xc = x - mean[..., None]
    var = (xc * xc).mean(axis=-1)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = xc * rstd[..., None]
    return xhat * gamma + beta, mean, rstd


def layernorm_bwd(dy: np.ndarray, x: np.ndarray, gamma: np.ndarray, mean: np.ndarray,
                  rstd: np.ndarray):
    """Vector-Jacobian product of ``layernorm_fwd``.

    With xhat = (x - mean) rstd and g = dy * gamma:
      dx = rstd (g - mean(g) - xhat mean(g xhat)),
      dgamma = sum over rows of dy * xhat, dbeta = sum over rows of dy.
    """
    xhat = (x - mean[..., None]) * rstd[..., None]
    g = dy * gamma
    dx = rstd[..., None] * (g - g.mean(axis=-1, keepdims=True)
                            - xhat * (g * xhat).mean(axis=-1, keepdims=True))
    dgamma = (dy * xhat).reshape(-1, x.shape[-1]).sum(axis=0)
    dbeta = dy.reshape(-1, x.shape[-1]).sum(axis=0)
    return dx, dgamma, dbeta


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Softmax along the last axis, max-subtracted; -inf entries get 0."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)
