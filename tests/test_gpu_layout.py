"""Bit-exact shard layouts on the GPU (tp_shard_* / tp_unshard_*) against the oracle's slicing."""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import require_gpu
from oracle import layout as olay

pytestmark = pytest.mark.gpu


def _bits(rows, cols, seed):
    g = np.random.default_rng(seed)
    return g.integers(0, 2 ** 16, size=(rows, cols), dtype=np.uint16)


def _dev(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def _host(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("rows,cols,t", [(256, 1024, 2), (3072, 12288, 8), (5, 24, 4), (7, 6, 2),
                                         (33, 40, 8), (1, 64, 1)])
def test_shard_cols_bit_exact(rows, cols, t):
    require_gpu()
    w = _bits(rows, cols, rows + cols)
    out = torch.empty(t, rows, cols // t, dtype=torch.bfloat16, device="cuda")
    tl.shard_cols(_dev(w), rows, cols, t, out)
    assert np.array_equal(_host(out), olay.shard_cols(w, t))
    back = torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda")
    tl.unshard_cols(out, rows, cols, t, back)
    assert np.array_equal(_host(back), w)


@pytest.mark.parametrize("rows,cols,t", [(1024, 256, 2), (12288, 3072, 8), (8, 5, 4)])
def test_shard_rows_bit_exact(rows, cols, t):
    require_gpu()
    w = _bits(rows, cols, 7)
    out = torch.empty(t, rows // t, cols, dtype=torch.bfloat16, device="cuda")
    tl.shard_rows(_dev(w), rows, cols, t, out)
    assert np.array_equal(_host(out), olay.shard_rows(w, t))


@pytest.mark.parametrize("rows,heads,dh,t", [(1024, 16, 64, 4), (4096, 32, 128, 8), (1, 16, 64, 4),
                                             (3, 8, 3, 2), (16, 4, 2, 4)])
def test_shard_qkv_heads_bit_exact(rows, heads, dh, t):
    require_gpu()
    D = heads * dh
    w = _bits(rows, 3 * D, heads)
    out = torch.empty(t, rows, 3 * D // t, dtype=torch.bfloat16, device="cuda")
    tl.shard_qkv_heads(_dev(w), rows, D, heads, t, out)
    assert np.array_equal(_host(out), olay.shard_qkv(w, t))
    back = torch.empty(rows, 3 * D, dtype=torch.bfloat16, device="cuda")
    tl.unshard_qkv_heads(out, rows, D, heads, t, back)
    assert np.array_equal(_host(back), w)
