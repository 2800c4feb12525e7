"""The reduction count does not depend on t ("The attention heads split":
one all-reduce per sublayer, two per block, whatever the tensor-parallel
degree; only the message size changes).

On one GPU each reduction is the K walk of a row-parallel product, inside
one GEMM launch.  The launch sequence of a sublayer's forward and backward
must therefore be the same for t = 1, 2, 4, 8, with no separate reduction
kernel: exactly one shard-summing product per sublayer per direction.
"""
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from synth import Workload, make_inputs
from tensor_transformer_layer_column_b200.sublayer import (ShardedAttention, ShardedLayer,
                                                           ShardedMLP)

pytestmark = pytest.mark.gpu

PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")


def _launches(kind, t):
    w = Workload("count", {"mlp": "mlp_fwdbwd", "attn": "attn_fwdbwd", "layer": "layer_fwdbwd"}[kind],
                 batch=2, seq=128, hidden=512, ffn=2048, heads=8, head_dim=64, t=t)
    g = dev(make_inputs(w, seed=11))
    d = dims_of(w)
    if kind == "mlp":
        m = ShardedMLP(d, g["w1"], g["b1"], g["w2"], g["b2"])
    elif kind == "attn":
        m = ShardedAttention(d, g["wqkv"], g["bqkv"], g["wout"], g["bout"])
    else:
        m = ShardedLayer(d, {k: g[k] for k in PARAMS})

    def step():
        m.forward(g["x"])
        m.backward(g["dy"])

    step()                                   # workspaces and descriptors set up outside the trace
    torch.cuda.synchronize()
    tr = tl.LaunchTrace(128)
    with tr:
        step()
    rec = tr.records()
    assert_no_device_error()
    assert tr.count == len(rec)
    return [k for k, _, _ in rec]


@pytest.mark.parametrize("kind", ["mlp", "attn", "layer"])
def test_launch_sequence_independent_of_t(kind):
    require_gpu()
    seqs = {t: _launches(kind, t) for t in (1, 2, 4, 8)}
    for t in (2, 4, 8):
        assert seqs[t] == seqs[1], (t, seqs[t], seqs[1])


def test_mlp_one_shard_sum_per_direction():
    """MLP: forward = column-parallel product + row-parallel product (shard sum
    in its K walk); backward = dA (its epilogue also writes db1's column
    partials, reduced right after), dW2, dW1 and the input-gradient product
    (shard sum in its K walk), then db2's two-pass column sum.  No other kernel."""
    require_gpu()
    seq = _launches("mlp", 8)
    assert seq == ["gemm", "gemm", "gemm", "colsum", "gemm", "gemm", "gemm",
                   "colsum", "colsum"]
