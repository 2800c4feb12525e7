"""Parity of the CUDA pre-LN layer (tp_layer_fwd / tp_layer_bwd) with the fp64 oracle.

"The layernorm placement the paper flags as critical": h = x + Attn(LN1(x));
y = h + MLP(LN2(h)), with both sublayers tensor-parallel over t shards.
"""
import numpy as np
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


def _run_and_compare(w, inp, reference=None):
    d = dims_of(w)
    g = dev(inp)
    layer = ShardedLayer(d, {k: g[k] for k in PARAMS})
    y, acts = layer.forward(g["x"])
    dx, grads = layer.backward(g["dy"])
    torch.cuda.synchronize()
    assert_no_device_error()
    t = w.t
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x = to_f64(inp["x"])
    if reference is None:
        yr, sv = olayer.layer_fwd(x, p, w.batch, w.heads, w.causal, w.ln_eps)
    else:
        yr, sv, gr = reference
    check("y", y, yr)
    check("h", acts["h"], sv["h"])
    check("u1", acts["u1"], sv["u1"])
    check("u2", acts["u2"], sv["u2"])
    check("o", acts["o"], olay.shard_cols(sv["o"], t))
    check("lse", acts["lse"], sv["lse"])
    check("a", acts["a"], olay.shard_cols(sv["a"], t))
    check("hact", acts["hact"], olay.shard_cols(sv["hact"], t))
    if reference is None:
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


@pytest.mark.parametrize("B,S,H,dh,F,t", [(2, 128, 4, 64, 1024, 2), (1, 200, 2, 128, 1024, 2),
                                          (2, 96, 8, 64, 2048, 8)])
@pytest.mark.parametrize("affine", [False, True])
def test_layer_fwd_bwd_small(B, S, H, dh, F, t, affine):
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=B, seq=S, hidden=H * dh, ffn=F, heads=H,
                 head_dim=dh, t=t)
    _run_and_compare(w, make_inputs(w, seed=13, random_affine=affine))


def test_layer_full_size_B4_S2048_D4096_H32_F16384_t8():
    """The pre-LN GPT layer at full size, every output and gradient against the full oracle."""
    require_gpu()
    from full_size_reference import pre_ln_layer
    w, inp, yr, sv, gr = pre_ln_layer()
    _run_and_compare(w, inp, reference=(yr, sv, gr))


# ---------------------------------------------------------------- post-LN layer

def _run_and_compare_postln(w, inp):
    d = dims_of(w)
    g = dev(inp)
    layer = ShardedLayer(d, {k: g[k] for k in PARAMS}, placement="post")
    y, acts = layer.forward(g["x"])
    dx, grads = layer.backward(g["dy"])
    torch.cuda.synchronize()
    assert_no_device_error()
    t = w.t
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x = to_f64(inp["x"])
    yr, sv = olayer.postln_layer_fwd(x, p, w.batch, w.heads, w.causal, w.ln_eps)
    check("y", y, yr)
    for k in ("z1", "h", "z2"):
        check(k, acts[k], sv[k])
    check("a", acts["a"], olay.shard_cols(sv["a"], t))
    gr = olayer.postln_layer_bwd(x, p, to_f64(inp["dy"]), w.batch, w.heads, w.causal, w.ln_eps)
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


@pytest.mark.parametrize("B,S,H,dh,F,t", [(2, 128, 4, 64, 1024, 2), (1, 200, 2, 128, 1024, 2),
                                          (2, 96, 8, 64, 2048, 8)])
@pytest.mark.parametrize("affine", [False, True])
def test_postln_layer_fwd_bwd_small(B, S, H, dh, F, t, affine):
    require_gpu()
    w = Workload("postln_test", "layer_fwdbwd", batch=B, seq=S, hidden=H * dh, ffn=F, heads=H,
                 head_dim=dh, t=t)
    _run_and_compare_postln(w, make_inputs(w, seed=17, random_affine=affine))


def test_postln_layer_full_size_B4_S2048_D4096_H32_F16384_t8():
    """The post-LN arm at the pre-LN layer's full size, every output and gradient."""
    require_gpu()
    w = workload("layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8")
    _run_and_compare_postln(w, make_inputs(w))


@pytest.mark.parametrize("placement", ["pre", "post"])
def test_layer_zero_tokens(placement):
    """batch 0: the forward does nothing and every parameter gradient is zero."""
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=0, seq=64, hidden=256, ffn=1024, heads=2,
                 head_dim=128, t=2)
    inp = make_inputs(w, seed=5)
    g = dev(inp)
    layer = ShardedLayer(dims_of(w), {k: g[k] for k in PARAMS}, placement=placement)
    layer.forward(g["x"])
    grads = layer.alloc_grads()
    for v in grads.values():
        v.fill_(1.0)
    layer.backward(g["dy"], grads=grads)
    torch.cuda.synchronize()
    assert_no_device_error()
    for k, v in grads.items():
        assert not v.float().abs().any(), k


def test_layer_kept_fp16_wqkv_equals_converting_again():
    """acts["wqkv16"] (the forward's fp16 copy of Wqkv, reused by the backward)
    gives the same y, dx and gradients, bit for bit, as leaving it NULL."""
    require_gpu()
    w = Workload("layer_test", "layer_fwdbwd", batch=2, seq=96, hidden=512, ffn=1024, heads=4,
                 head_dim=128, t=4)
    inp = make_inputs(w, seed=19, random_affine=True)
    g = dev(inp)
    out = []
    for keep in (True, False):
        layer = ShardedLayer(dims_of(w), {k: g[k] for k in PARAMS})
        acts = layer.alloc_acts()
        if not keep:
            acts["wqkv16"] = None
        y, _ = layer.forward(g["x"], acts=acts) if keep else _forward_without_copy(layer, g, acts)
        dx, grads = layer.backward(g["dy"])
        torch.cuda.synchronize()
        assert_no_device_error()
        out.append((y.clone(), dx.clone(), {k: v.clone() for k, v in grads.items()}))
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
    for k in out[0][2]:
        assert torch.equal(out[0][2][k], out[1][2][k]), k


def _forward_without_copy(layer, g, acts):
    """The layer forward through the binding with acts["wqkv16"] = NULL."""
    import tensor_transformer_layer_column_b200 as tl
    from tensor_transformer_layer_column_b200.sublayer import OP_LAYER_FWD, _ws
    d = layer.dims
    y = torch.empty_like(g["x"])
    layer.ws_fwd = _ws(OP_LAYER_FWD, d, layer.device)
    tl.layer_fwd(d, g["x"], layer.p, acts, y, layer.ws_fwd)
    layer.saved = (g["x"], acts)
    return y, acts
