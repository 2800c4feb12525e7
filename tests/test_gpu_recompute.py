"""Activation recomputation for the pre-LN layer (tp_layer_fwd_nosave /
tp_layer_bwd_recompute).

"What actually limits throughput in production", the activation memory vs.
recomputation trade-off: the activations are computed again in the backward
pass instead of being kept.  The recomputing path launches the same kernels on
the same inputs as the path that saves them, and the library is deterministic,
so y, dx and every parameter gradient must agree with the saving path bit for
bit; the saving path is itself held to the fp64 oracle (test_gpu_layer.py), and
one case here checks the recomputing path against the oracle directly.
"""
import pytest
import torch

from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import layer as olayer
from oracle import layout as olay
from parity import check
from synth import Workload, make_inputs, to_f64, workload
from tensor_transformer_layer_column_b200.sublayer import ShardedLayer

pytestmark = pytest.mark.gpu

PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")
GRADS = ("dln1_g", "dln1_b", "dwqkv", "dbqkv", "dwout", "dbout", "dln2_g", "dln2_b", "dw1", "db1",
         "dw2", "db2")


def _both_paths(w, inp):
    d = dims_of(w)
    g = dev(inp)
    p = {k: g[k] for k in PARAMS}
    saving = ShardedLayer(d, p)
    y0, _ = saving.forward(g["x"])
    dx0, gr0 = saving.backward(g["dy"])
    rec = ShardedLayer(d, p, recompute=True)
    y1, acts = rec.forward(g["x"])
    assert acts is None
    dx1, gr1 = rec.backward(g["dy"])
    torch.cuda.synchronize()
    assert_no_device_error()
    return (y0, dx0, gr0), (y1, dx1, gr1)


def _assert_bitwise(a, b):
    (y0, dx0, gr0), (y1, dx1, gr1) = a, b
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16)), "y differs"
    assert torch.equal(dx0.view(torch.int16), dx1.view(torch.int16)), "dx differs"
    for k in GRADS:
        assert torch.equal(gr0[k].view(torch.int16), gr1[k].view(torch.int16)), f"{k} differs"


@pytest.mark.parametrize("B,S,H,dh,F,t", [(2, 128, 4, 64, 1024, 2), (1, 200, 2, 128, 1024, 2),
                                          (2, 96, 8, 64, 2048, 8)])
@pytest.mark.parametrize("affine", [False, True])
def test_recompute_matches_saving_path_bitwise(B, S, H, dh, F, t, affine):
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=B, seq=S, hidden=H * dh, ffn=F, heads=H,
                 head_dim=dh, t=t)
    a, b = _both_paths(w, make_inputs(w, seed=23, random_affine=affine))
    _assert_bitwise(a, b)


def test_recompute_against_oracle():
    """The recomputing path on its own against the fp64 oracle (ragged S, t=2)."""
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=1, seq=200, hidden=256, ffn=1024, heads=2,
                 head_dim=128, t=2)
    inp = make_inputs(w, seed=29, random_affine=True)
    d = dims_of(w)
    g = dev(inp)
    layer = ShardedLayer(d, {k: g[k] for k in PARAMS}, recompute=True)
    y, _ = layer.forward(g["x"])
    dx, grads = layer.backward(g["dy"])
    torch.cuda.synchronize()
    assert_no_device_error()
    t = w.t
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x = to_f64(inp["x"])
    yr, _ = olayer.layer_fwd(x, p, w.batch, w.heads, w.causal, w.ln_eps)
    check("y", y, yr)
    gr = olayer.layer_bwd(x, p, to_f64(inp["dy"]), w.batch, w.heads, w.causal, w.ln_eps)
    check("dx", dx, gr["dx"])
    check("dwqkv", grads["dwqkv"], olay.shard_qkv(gr["dwqkv"], t))
    check("dbqkv", grads["dbqkv"], olay.shard_qkv(gr["dbqkv"][None, :], t))
    check("dwout", grads["dwout"], olay.shard_rows(gr["dwout"], t))
    check("dbout", grads["dbout"], gr["dbout"])
    check("dw1", grads["dw1"], olay.shard_cols(gr["dw1"], t))
    check("db1", grads["db1"], gr["db1"])
    check("dw2", grads["dw2"], olay.shard_rows(gr["dw2"], t))
    check("db2", grads["db2"], gr["db2"])
    for k in ("dln1_g", "dln1_b", "dln2_g", "dln2_b"):
        check(k, grads[k], gr[k])


def test_recompute_zero_tokens():
    """Zero tokens: every parameter gradient is zero, nothing else is touched."""
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=0, seq=64, hidden=256, ffn=1024, heads=2,
                 head_dim=128, t=2)
    inp = make_inputs(w, seed=3)
    d = dims_of(w)
    g = dev(inp)
    layer = ShardedLayer(d, {k: g[k] for k in PARAMS}, recompute=True)
    layer.forward(g["x"])
    grads = layer.alloc_grads()
    for v in grads.values():
        v.fill_(1.0)
    layer.backward(g["dy"], grads=grads)
    torch.cuda.synchronize()
    assert_no_device_error()
    for k in GRADS:
        assert not grads[k].float().abs().any(), k


def test_recompute_full_size_B4_S2048_D4096_H32_F16384_t8():
    """The full pre-LN layer size: bitwise agreement with the saving path, and
    no activations held between the passes."""
    require_gpu()
    w = workload("layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8")
    a, b = _both_paths(w, make_inputs(w))
    _assert_bitwise(a, b)
