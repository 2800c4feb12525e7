"""Parity of the CUDA attention sublayer (tp_attn_fwd / tp_attn_bwd) with the fp64 oracle.

"The attention heads split": Q, K, V split column-wise by head, full attention
per head on its shard, Wout split by rows and the partial outputs summed.
"""
import numpy as np
import pytest
import torch

from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import attention as oatt
from oracle import layout as olay
from parity import check
from synth import Workload, make_inputs, to_f64, workload
import tensor_transformer_layer_column_b200 as tl
from tensor_transformer_layer_column_b200.sublayer import ShardedAttention

pytestmark = pytest.mark.gpu


def _run(w, inp, backward):
    d = dims_of(w)
    g = dev(inp)
    m = ShardedAttention(d, g["wqkv"], g["bqkv"], g["wout"], g["bout"])
    o = m.forward(g["x"], resid=g.get("resid"))
    grads = m.backward(g["dy"]) if backward else None
    torch.cuda.synchronize()
    assert_no_device_error()
    return o, grads


def _compare(w, inp, o, grads):
    t = w.t
    x, wqkv, bqkv, wout, bout = (to_f64(inp[k]) for k in ("x", "wqkv", "bqkv", "wout", "bout"))
    resid = to_f64(inp["resid"]) if "resid" in inp else None
    y, sv = oatt.attn_fwd(x, wqkv, bqkv, wout, bout, w.batch, w.heads, w.causal, resid=resid)
    check("y", o["y"], y)
    check("qkv_save", o["qkv"], olay.shard_qkv(sv["qkv"], t))
    check("o_save", o["o"], olay.shard_cols(sv["o"], t))
    check("lse", o["lse"], sv["lse"])
    if grads is not None:
        g = oatt.attn_bwd(x, wqkv, bqkv, wout, to_f64(inp["dy"]), w.batch, w.heads, w.causal)
        check("dx", grads["dx"], g["dx"])
        check("dwqkv", grads["dwqkv"], olay.shard_qkv(g["dwqkv"], t))
        check("dbqkv", grads["dbqkv"], olay.shard_qkv(g["dbqkv"][None, :], t))
        check("dwout", grads["dwout"], olay.shard_rows(g["dwout"], t))
        check("dbout", grads["dbout"], g["dbout"])


def test_attn_fwd_workload_B4_S1024_D1024_H16_t4():
    require_gpu()
    w = workload("attn_fwd_B4_S1024_D1024_H16_t4")
    inp = make_inputs(w)
    o, _ = _run(w, inp, backward=False)
    _compare(w, inp, o, None)


# Sequence lengths that are not multiples of the 128/64 tiles, both head
# dims, causal and full masks, every t.
SMALL = [
    (2, 100, 4, 64, 2, True),
    (1, 300, 8, 128, 4, True),
    (2, 64, 2, 64, 1, False),
    (1, 257, 8, 64, 8, True),
    (3, 130, 4, 128, 2, False),
    (2, 512, 4, 128, 4, True),
    (1, 1, 2, 64, 2, True),
]


@pytest.mark.parametrize("B,S,H,dh,t,causal", SMALL)
@pytest.mark.parametrize("affine", [False, True])
def test_attn_fwd_bwd_small(B, S, H, dh, t, causal, affine):
    require_gpu()
    w = Workload("attn_test", "attn_fwdbwd", batch=B, seq=S, hidden=H * dh, heads=H,
                 head_dim=dh, t=t, causal=causal)
    inp = make_inputs(w, seed=7, random_affine=affine)
    o, grads = _run(w, inp, backward=True)
    _compare(w, inp, o, grads)


# More (key block, head, batch) items than SMs, so that each CTA of the
# persistent dK/dV kernel walks several items of different lengths (causal:
# 5, 3 and 1 query blocks of 64 at S = 300) and the stage ring, the score
# buffers and the accumulator hand-over carry from one item to the next.
MANY_ITEMS = [
    (4, 300, 32, 64, 4, True),
    (2, 200, 48, 128, 8, False),
]


@pytest.mark.parametrize("B,S,H,dh,t,causal", MANY_ITEMS)
def test_attn_fwd_bwd_more_items_than_sms(B, S, H, dh, t, causal):
    require_gpu()
    w = Workload("attn_test", "attn_fwdbwd", batch=B, seq=S, hidden=H * dh, heads=H,
                 head_dim=dh, t=t, causal=causal)
    inp = make_inputs(w, seed=13, random_affine=True)
    o, grads = _run(w, inp, backward=True)
    _compare(w, inp, o, grads)
    # The walk over several items per CTA keeps the results run-to-run identical.
    o2, grads2 = _run(w, inp, backward=True)
    for k in o:
        assert torch.equal(o[k], o2[k]), k
    for k in grads:
        assert torch.equal(grads[k], grads2[k]), k


def test_attn_deterministic_run_to_run():
    require_gpu()
    w = Workload("attn_test", "attn_fwdbwd", batch=2, seq=384, hidden=512, heads=4, head_dim=128,
                 t=4)
    inp = make_inputs(w, seed=9, random_affine=True)
    o1, g1 = _run(w, inp, True)
    o2, g2 = _run(w, inp, True)
    for k in o1:
        assert torch.equal(o1[k], o2[k]), k
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


@pytest.fixture
def recompute_dq():
    prev = tl.attn_set_ds_limit(0)
    yield
    tl.attn_set_ds_limit(prev)


# With the dS^T limit at 0 the dq kernel recomputes q k^T and dO v^T instead
# of reading dS^T back (the path problems too large to keep dS^T take).
@pytest.mark.parametrize("B,S,H,dh,t,causal", SMALL[:6] + MANY_ITEMS)
def test_attn_bwd_recomputed_scores_dq(B, S, H, dh, t, causal, recompute_dq):
    require_gpu()
    w = Workload("attn_test", "attn_fwdbwd", batch=B, seq=S, hidden=H * dh, heads=H,
                 head_dim=dh, t=t, causal=causal)
    inp = make_inputs(w, seed=11, random_affine=True)
    o, grads = _run(w, inp, backward=True)
    _compare(w, inp, o, grads)
