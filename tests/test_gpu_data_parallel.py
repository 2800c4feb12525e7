"""The data-parallel gradient path on the GPU.

tp_layer_bwd_notify is tp_layer_bwd plus three events, one per group of
parameter gradients ("3D decomposition in practice": the replicas' gradient
all-reduce starts while the backward still computes).  Checked here: its
results equal tp_layer_bwd's bit for bit and every event completes; and the
bucketed reducer, on a one-rank NCCL group (one GPU), issues its collectives
behind those events and leaves the gradients as a one-replica sum or average
leaves them (unchanged), with the layer writing straight into the buckets.
"""
import socket

import pytest
import torch
import torch.distributed as dist

from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from synth import Workload, make_inputs
from tensor_transformer_layer_column_b200.data_parallel import (GradientAllReduce,
                                                                sharded_layer_buckets)
from tensor_transformer_layer_column_b200.sublayer import ShardedLayer

pytestmark = pytest.mark.gpu
PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2",
          "b2")


def _layer():
    w = Workload("dp_gpu", "layer_fwdbwd", batch=2, seq=128, hidden=512, ffn=2048, heads=4,
                 head_dim=128, t=4)
    inp = make_inputs(w, seed=31, random_affine=True)
    g = dev(inp)
    layer = ShardedLayer(dims_of(w), {k: g[k] for k in PARAMS})
    return layer, g


def _events():
    ev = {}
    for k in ("mlp", "attn", "ln1"):
        e = torch.cuda.Event()
        e.record()
        ev[k] = e
    return ev


def test_notify_backward_equals_plain_backward_and_records_every_event():
    require_gpu()
    layer, g = _layer()
    layer.forward(g["x"])
    dx0, g0 = layer.backward(g["dy"])
    dx0, g0 = dx0.clone(), {k: v.clone() for k, v in g0.items()}
    ev = _events()
    torch.cuda.synchronize()
    dx1, g1 = layer.backward(g["dy"], ready=ev)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert all(e.query() for e in ev.values())
    assert torch.equal(dx1, dx0)
    for k in g0:
        assert torch.equal(g1[k], g0[k]), k


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("average", [False, True])
def test_bucketed_allreduce_on_a_one_rank_nccl_group(average):
    require_gpu()
    layer, g = _layer()
    layer.forward(g["x"])
    dx_ref, g_ref = layer.backward(g["dy"])
    g_ref = {k: v.clone() for k, v in g_ref.items()}
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        buckets, grads = sharded_layer_buckets(layer)
        reducer = GradientAllReduce(buckets, average=average)
        ev = reducer.events()
        for _ in range(2):                       # two steps through the same buckets
            layer.backward(g["dy"], grads=grads, ready=ev)
            for name in ("mlp", "attn", "ln1"):
                reducer.launch(name, ev[name])
            reducer.finish()
        torch.cuda.synchronize()
        assert_no_device_error()
        assert reducer.order == ["mlp", "attn", "ln1"] * 2
        for k, v in g_ref.items():
            assert torch.equal(grads[k], v), k
    finally:
        dist.destroy_process_group()
