"""Shared helpers of the -m gpu tests (device inputs from the seeded generator)."""
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip("needs an sm_100 device")
    tl.lib()   # raises if the library is missing: no silent fallback


def dev(inputs):
    return {k: v.cuda() for k, v in inputs.items()}


def dims_of(w, ln_eps=1e-5):
    return tl.Dims.of(w.batch, w.seq, w.hidden, w.ffn, w.heads, w.head_dim, w.t,
                      1 if w.causal else 0, ln_eps)


def assert_no_device_error():
    assert tl.check_error() == 0
