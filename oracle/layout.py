"""Shard-packed weight layouts (NumPy; any dtype, so bf16 bit patterns work).

Test infrastructure only (see the package docstring).

The pages define the slicing ("How transformer layers actually decompose",
"The attention heads split"):
* the first matrix of each pair (W1, and Q, K, V) is split by COLUMNS into t
  contiguous blocks, shard i owning block i ("[W1_left | W1_right]");
* the second matrix (W2, Wout) is split by ROWS ("[W2_top; W2_bottom]");
* for attention, shard i owns the columns of heads i*H/t .. (i+1)*H/t - 1.
Packed layouts: column shards as [t][rows][cols/t]; row shards as
[t][rows/t][cols] (byte-identical to the unsharded matrix); the fused
[D, 3D] = [Wq | Wk | Wv] matrix as [t][rows][3 D/t] with shard i =
[Wq_i | Wk_i | Wv_i].
"""
from __future__ import annotations

import numpy as np


def shard_cols(w: np.ndarray, t: int) -> np.ndarray:
    rows, cols = w.shape
    if cols % t:
        raise ValueError("columns not divisible by t")
    return np.stack([w[:, i * (cols // t):(i + 1) * (cols // t)] for i in range(t)])


def unshard_cols(p: np.ndarray) -> np.ndarray:
    return np.concatenate(list(p), axis=1)


def shard_rows(w: np.ndarray, t: int) -> np.ndarray:
    rows, cols = w.shape
    if rows % t:
        raise ValueError("rows not divisible by t")
    return np.stack([w[i * (rows // t):(i + 1) * (rows // t), :] for i in range(t)])


def unshard_rows(p: np.ndarray) -> np.ndarray:
    return np.concatenate(list(p), axis=0)


def shard_qkv(w: np.ndarray, t: int) -> np.ndarray:
    """[rows, 3D] = [Wq | Wk | Wv] -> [t][rows][3 D/t], shard i = [Wq_i | Wk_i | Wv_i]."""
    rows, c3 = w.shape
    d = c3 // 3
    if c3 % 3 or d % t:
        raise ValueError("bad fused QKV width")
    dt = d // t
    return np.stack([np.concatenate([w[:, j * d + i * dt:j * d + (i + 1) * dt] for j in range(3)],
                                    axis=1) for i in range(t)])


def unshard_qkv(p: np.ndarray) -> np.ndarray:
    t, rows, c3t = p.shape
    dt = c3t // 3
    return np.concatenate([p[i][:, j * dt:(j + 1) * dt] for j in range(3) for i in range(t)],
                          axis=1)
