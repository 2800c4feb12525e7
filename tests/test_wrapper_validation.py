"""The torch-facing wrappers check every tensor argument (dtype, shape,
device) before anything reaches the C ABI, which takes raw pointers and so
cannot tell a wrong buffer from a right one.  CPU only: each case fails
before any device is touched."""
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from tensor_transformer_layer_column_b200.sublayer import (ShardedAttention, ShardedLayer,
                                                           ShardedMLP)

BF = torch.bfloat16
D, F, H, DH, T = 256, 1024, 2, 128, 8
DIMS = tl.Dims.of(1, T, D, F, H, DH, 2)


def z(*shape, dtype=BF):
    return torch.zeros(*shape, dtype=dtype)


def test_mlp_weights_checked():
    with pytest.raises(ValueError, match=r"w1: shape \(1024, 256\), expected \(256, 1024\)"):
        ShardedMLP(DIMS, z(F, D), None, z(F, D), None)
    with pytest.raises(ValueError, match="w2: dtype torch.float32"):
        ShardedMLP(DIMS, z(D, F), None, z(F, D, dtype=torch.float32), None)
    with pytest.raises(ValueError, match=r"b1: shape \(256,\)"):
        ShardedMLP(DIMS, z(D, F), z(D), z(F, D), None)
    with pytest.raises(ValueError, match="CUDA"):
        ShardedMLP(DIMS, z(D, F), z(F), z(F, D), z(D))        # right shapes, but host tensors


def test_attention_weights_checked():
    with pytest.raises(ValueError, match=r"wqkv: shape \(256, 256\)"):
        ShardedAttention(DIMS, z(D, D), None, z(D, D), None)
    with pytest.raises(ValueError, match=r"bqkv: shape \(256,\)"):
        ShardedAttention(DIMS, z(D, 3 * D), z(D), z(D, D), None)
    with pytest.raises(ValueError, match="CUDA"):
        ShardedAttention(DIMS, z(D, 3 * D), z(3 * D), z(D, D), z(D))


def _params():
    return {"ln1_g": z(D), "ln1_b": z(D), "wqkv": z(D, 3 * D), "bqkv": z(3 * D),
            "wout": z(D, D), "bout": z(D), "ln2_g": z(D), "ln2_b": z(D), "w1": z(D, F),
            "b1": z(F), "w2": z(F, D), "b2": z(D)}


def test_layer_parameters_checked():
    p = _params()
    del p["ln2_g"]
    with pytest.raises(ValueError, match=r"p\['ln2_g'\] is required"):
        ShardedLayer(DIMS, p)
    p = _params()
    p["w2"] = z(D, F)
    with pytest.raises(ValueError, match=r"p\['w2'\]: shape \(256, 1024\), expected \(1024, 256\)"):
        ShardedLayer(DIMS, p)
    p = _params()
    p["bqkv"] = None                                         # optional biases may be absent
    with pytest.raises(ValueError, match="CUDA"):
        ShardedLayer(DIMS, p)
