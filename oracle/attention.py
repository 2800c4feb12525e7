"""Unsharded causal multi-head self-attention sublayer (fp64 NumPy).

Test infrastructure only (see the package docstring).

Definition ("The attention heads split": H independent heads, each with its
own Q, K, V projections; an output projection):
    [q | k | v] = x Wqkv + bqkv, Wqkv [D, 3D] = [Wq | Wk | Wv];
    head h uses columns h*dh .. (h+1)*dh - 1 of each of q, k, v;
    O_h = softmax(q_h k_h^T / sqrt(dh) + M) v_h, M[s, s'] = -inf for s' > s;
    y = concat_h(O_h) Wout + bout (+ r).
Readings where the pages are silent: the 1/sqrt(dh) score scale, the causal
mask includes the diagonal and stays within one batch element, the fused
Wqkv column order [Wq | Wk | Wv].  Rows of x are batch-outer: row b*S + s.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .core import softmax_rows


def _heads(m: np.ndarray, batch: int, seq: int, heads: int) -> np.ndarray:
    """[T, H*dh] -> [B, H, S, dh]."""
    dh = m.shape[1] // heads
    return m.reshape(batch, seq, heads, dh).transpose(0, 2, 1, 3)


def _unheads(m: np.ndarray) -> np.ndarray:
    """[B, H, S, dh] -> [T, H*dh]."""
    b, h, s, dh = m.shape
    return m.transpose(0, 2, 1, 3).reshape(b * s, h * dh)


def _scores(q, k, causal: bool):
    """q k^T / sqrt(dh) with the causal mask, for one batch element [H, S, dh]."""
    dh = q.shape[-1]
    s = q @ k.transpose(0, 2, 1) / np.sqrt(dh)
    if causal:
        seq = q.shape[1]
        s = np.where(np.tril(np.ones((seq, seq), dtype=bool)), s, -np.inf)
    return s


def attn_core_fwd(q, k, v, causal: bool = True):
    """Per-head attention for [B, H, S, dh] inputs.

    Returns (O [B, H, S, dh], lse [B, H, S]) where lse is the natural log of
    the softmax denominator of the scaled, masked scores.
    """
    o = np.empty_like(q)
    lse = np.empty(q.shape[:3])
    for b in range(q.shape[0]):
        s = _scores(q[b], k[b], causal)
        m = s.max(axis=-1, keepdims=True)
        lse[b] = (m + np.log(np.exp(s - m).sum(axis=-1, keepdims=True)))[..., 0]
        o[b] = softmax_rows(s) @ v[b]
    return o, lse


def attn_core_bwd(q, k, v, do, causal: bool = True):
    """Vector-Jacobian product of ``attn_core_fwd`` (O only) for dO.

    P = softmax(S), O = P v:
      dv = P^T dO,  dP = dO v^T,  dS = P * (dP - rowsum(dP * P)),
      dq = dS k / sqrt(dh),  dk = dS^T q / sqrt(dh).
    """
    dh = q.shape[-1]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(q.shape[0]):
        p = softmax_rows(_scores(q[b], k[b], causal))
        dv[b] = p.transpose(0, 2, 1) @ do[b]
        dp = do[b] @ v[b].transpose(0, 2, 1)
        ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
        dq[b] = ds @ k[b] / np.sqrt(dh)
        dk[b] = ds.transpose(0, 2, 1) @ q[b] / np.sqrt(dh)
    return dq, dk, dv


def attn_fwd(x, wqkv, bqkv, wout, bout, batch: int, heads: int, causal: bool = True,
             resid: Optional[np.ndarray] = None):
    """Returns (y, saved) with saved = {qkv [T, 3D], o [T, D], lse [B, H, S]}."""
    T, D = x.shape
    seq = T // batch
    qkv = x @ wqkv + bqkv
    q, k, v = (_heads(qkv[:, i * D:(i + 1) * D], batch, seq, heads) for i in range(3))
    o4, lse = attn_core_fwd(q, k, v, causal)
    o = _unheads(o4)
    y = o @ wout + bout
    if resid is not None:
        y = y + resid
    return y, {"qkv": qkv, "o": o, "lse": lse}


def attn_bwd(x, wqkv, bqkv, wout, dy, batch: int, heads: int, causal: bool = True):
    """Vector-Jacobian product of ``attn_fwd`` for upstream gradient dy.

    Returns a dict with dx, dwqkv, dbqkv, dwout, dbout (the residual input's
    gradient is dy itself and is not returned).
    """
    T, D = x.shape
    seq = T // batch
    qkv = x @ wqkv + bqkv
    q, k, v = (_heads(qkv[:, i * D:(i + 1) * D], batch, seq, heads) for i in range(3))
    o4, _ = attn_core_fwd(q, k, v, causal)
    o = _unheads(o4)
    do = dy @ wout.T
    dq, dk, dv = attn_core_bwd(q, k, v, _heads(do, batch, seq, heads), causal)
    dqkv = np.concatenate([_unheads(dq), _unheads(dk), _unheads(dv)], axis=1)
    return {
        "dx": dqkv @ wqkv.T,
        "dwqkv": x.T @ dqkv,
        "dbqkv": dqkv.sum(axis=0),
        "dwout": o.T @ dy,
        "dbout": dy.sum(axis=0),
        "dqkv": dqkv,
        "do": do,
    }
