"""The tensor-parallel method itself, step by step, on t shards (fp64 NumPy).

Test infrastructure only (see the package docstring).  These functions follow
the pages' description of what each of the t GPUs does, in their order, and
exist to pin that the sharded computation re-associates the unsharded
definition exactly (up to fp64 rounding order).

MLP ("How transformer layers actually decompose"):
  1. W1 split column-wise, shard i computes GeLU(x W1_i) -- GeLU is applied
     locally because it is elementwise and each shard holds whole columns;
  2. W2 split row-wise, shard i computes the partial GeLU(x W1_i) W2_i;
  3. the partials are summed (one all-reduce).
Backward: shard i's weight gradients are local; the input gradient is the sum
over shards of dA_i W1_i^T (the backward all-reduce, "One Idea, Two
Insertions").

Attention ("The attention heads split"): shard i owns heads i*H/t ..
(i+1)*H/t - 1, i.e. those columns of Wq, Wk, Wv, computes full attention for
them, multiplies by its row block of Wout and the partials are summed.

Biases of the column-split matrices are split with their columns; the bias of
the row-split matrix is added once, after the sum.
"""
from __future__ import annotations

import numpy as np

from .attention import _heads, _unheads, attn_core_bwd, attn_core_fwd
from .core import gelu, gelu_grad


def mlp_fwd_sharded(x, w1, b1, w2, b2, t: int):
    F = w1.shape[1]
    ft = F // t
    y = 0.0
    for i in range(t):
        cols = slice(i * ft, (i + 1) * ft)
        h_i = gelu(x @ w1[:, cols] + b1[cols])      # column-parallel, local GeLU
        y = y + h_i @ w2[cols, :]                   # row-parallel partial sum
    return y + b2


def mlp_bwd_sharded(x, w1, b1, w2, dy, t: int):
    F = w1.shape[1]
    ft = F // t
    dx = 0.0
    dw1, db1, dw2 = np.empty_like(w1), np.empty_like(b1), np.empty_like(w2)
    for i in range(t):
        cols = slice(i * ft, (i + 1) * ft)
        a_i = x @ w1[:, cols] + b1[cols]
        da_i = (dy @ w2[cols, :].T) * gelu_grad(a_i)
        dw2[cols, :] = gelu(a_i).T @ dy
        dw1[:, cols] = x.T @ da_i
        db1[cols] = da_i.sum(axis=0)
        dx = dx + da_i @ w1[:, cols].T              # input-gradient reduction
    return {"dx": dx, "dw1": dw1, "db1": db1, "dw2": dw2, "db2": dy.sum(axis=0)}


def _shard_heads(x, wqkv, bqkv, i, t, batch, heads):
    T, D = x.shape
    dt = D // t
    seq = T // batch
    proj = []
    for j in range(3):
        cols = slice(j * D + i * dt, j * D + (i + 1) * dt)
        proj.append(_heads(x @ wqkv[:, cols] + bqkv[cols], batch, seq, heads // t))
    return proj


def attn_fwd_sharded(x, wqkv, bqkv, wout, bout, batch: int, heads: int, t: int,
                     causal: bool = True):
    D = x.shape[1]
    dt = D // t
    y = 0.0
    for i in range(t):
        q, k, v = _shard_heads(x, wqkv, bqkv, i, t, batch, heads)
        o_i, _ = attn_core_fwd(q, k, v, causal)         # local heads, no communication
        y = y + _unheads(o_i) @ wout[i * dt:(i + 1) * dt, :]
    return y + bout


def attn_bwd_sharded(x, wqkv, bqkv, wout, dy, batch: int, heads: int, t: int,
                     causal: bool = True):
    T, D = x.shape
    dt = D // t
    seq = T // batch
    dx = 0.0
    dwqkv, dbqkv, dwout = np.empty_like(wqkv), np.empty_like(bqkv), np.empty_like(wout)
    for i in range(t):
        rows = slice(i * dt, (i + 1) * dt)
        q, k, v = _shard_heads(x, wqkv, bqkv, i, t, batch, heads)
        o_i, _ = attn_core_fwd(q, k, v, causal)
        dwout[rows, :] = _unheads(o_i).T @ dy
        do_i = _heads(dy @ wout[rows, :].T, batch, seq, heads // t)
        grads = attn_core_bwd(q, k, v, do_i, causal)
        for j in range(3):
            cols = slice(j * D + i * dt, j * D + (i + 1) * dt)
            g = _unheads(grads[j])
            dwqkv[:, cols] = x.T @ g
            dbqkv[cols] = g.sum(axis=0)
            dx = dx + g @ wqkv[:, cols].T             # input-gradient reduction
    return {"dx": dx, "dwqkv": dwqkv, "dbqkv": dbqkv, "dwout": dwout,
            "dbout": dy.sum(axis=0)}
