"""Data-parallel gradient all-reduce (CPU only, gloo ranks).

"3D decomposition in practice" (blog): replicas of the layer train on
different batches and all-reduce their parameter gradients, off the critical
path.  These tests pin the host logic of data_parallel.GradBuckets /
GradientAllReduce: the bucket layout the library writes into, the groups
being reduced in the order the backward finishes them, sum and average, and
the composition with the one-shard-per-GPU driver (a 2 x 2 grid: two
tensor-parallel ranks per replica, two replicas), whose every gradient must
equal the oracle's gradient averaged over the two replicas' batches.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tensor_transformer_layer_column_b200.data_parallel import LAYER_GROUPS, GradBuckets


def test_bucket_views_are_aligned_slices_of_one_buffer_per_group():
    shapes = {"w1": (32, 16), "b1": (16,), "w2": (16, 32), "b2": (32,), "wqkv": (32, 48),
              "bqkv": (48,), "wout": (16, 32), "bout": (32,), "ln2_g": (32,), "ln2_b": (32,),
              "ln1_g": (32,), "ln1_b": (32,)}
    b = GradBuckets(shapes, LAYER_GROUPS, dtype=torch.float32, device="cpu")
    assert set(b.flat) == {"mlp", "attn", "ln1"}
    for g, names in LAYER_GROUPS.items():
        base = b.flat[g].data_ptr()
        for n in names:
            v = b.views[n]
            assert tuple(v.shape) == shapes[n] and v.is_contiguous()
            off = v.data_ptr() - base
            assert off % 256 == 0 and off + v.numel() * 4 <= b.flat[g].numel() * 4
    # Views of a group do not overlap: writing one leaves the others zero.
    b.views["w1"].fill_(1.0)
    assert b.flat["mlp"].sum() == 32 * 16 and not b.views["b1"].any()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import datetime
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, os.path.dirname(here))
    sys.path.insert(0, here)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))


def _spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out, key=lambda o: o[0])


def _sum_worker(rank, world, port, q, average):
    _init(rank, world, port)
    try:
        from tensor_transformer_layer_column_b200.data_parallel import (GradBuckets,
                                                                        GradientAllReduce)
        shapes = {"w1": (4, 8), "b1": (8,), "wqkv": (4, 12), "ln1_g": (4,)}
        b = GradBuckets(shapes, LAYER_GROUPS, dtype=torch.float64, device="cpu")
        for i, (n, v) in enumerate(sorted(b.views.items())):
            v.copy_(torch.arange(v.numel(), dtype=torch.float64).view(v.shape) * (rank + 1) + i)
        r = GradientAllReduce(b, average=average)
        for g in ("mlp", "attn", "ln1"):
            r.launch(g)
        r.finish()
        q.put((rank, {n: v.numpy().copy() for n, v in b.views.items()}, list(r.order)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("average", [False, True])
def test_groups_are_summed_or_averaged_over_two_replicas(average):
    out = _spawn(_sum_worker, 2, average)
    for rank, views, order in out:
        assert order == ["mlp", "attn", "ln1"]
        for i, (n, v) in enumerate(sorted(views.items())):
            base = np.arange(v.size, dtype=np.float64).reshape(v.shape)
            want = base * (1 + 2) + 2 * i          # ranks 0 and 1 contribute (r + 1) base + i
            if average:
                want = want / 2
            np.testing.assert_array_equal(v, want)
        np.testing.assert_array_equal(out[0][1]["w1"], out[1][1]["w1"])


PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2",
          "b2")


def _batch(dp):
    from synth import Workload, make_inputs, to_f64
    w = Workload("dp_host", "layer_fwdbwd", batch=2, seq=8, hidden=32, ffn=64, heads=4,
                 head_dim=8, t=2)
    params = make_inputs(w, seed=7, random_affine=True)          # the same weights everywhere
    data = make_inputs(w, seed=100 + dp)                         # each replica its own batch
    p64 = {k: to_f64(params[k]) for k in PARAMS}
    return w, p64, to_f64(data["x"]), to_f64(data["dy"])


def _grid_worker(rank, world, port, q):
    """Ranks laid out as (replica dp, tensor rank tp) = divmod(rank, 2)."""
    _init(rank, world, port)
    try:
        import tensor_transformer_layer_column_b200 as tl
        from tensor_transformer_layer_column_b200.data_parallel import (GradBuckets,
                                                                        GradientAllReduce)
        from tensor_transformer_layer_column_b200.tensor_parallel import (AllReduce, RankLayer,
                                                                          layer_backward,
                                                                          layer_forward,
                                                                          shard_shapes)
        from tp_cpu_ops import OracleRankOps, rank_params
        dp, tp = divmod(rank, 2)
        tp_groups = [dist.new_group([0, 1]), dist.new_group([2, 3])]
        dp_groups = [dist.new_group([0, 2]), dist.new_group([1, 3])]
        w, p64, x, dy = _batch(dp)
        dims = tl.Dims.of(w.batch, w.seq, w.hidden, w.ffn, w.heads, w.head_dim, w.t, 1, w.ln_eps)
        buckets = GradBuckets(shard_shapes(dims), LAYER_GROUPS, dtype=torch.float64, device="cpu")
        layer = RankLayer(dims, tp, rank_params(p64, dims, tp), OracleRankOps(dims),
                          grads=buckets.grads())
        reducer = GradientAllReduce(buckets, group=dp_groups[tp], average=True)
        ex = AllReduce(tp_groups[dp])
        layer_forward([layer], torch.from_numpy(x), ex)
        layer_backward([layer], torch.from_numpy(dy), ex, on_grads_ready=reducer.mark)
        reducer.finish()
        q.put((rank, {k: v.numpy().copy() for k, v in layer.grads.items()}, list(reducer.order)))
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_times_data_parallel_grid_of_four_ranks():
    from oracle import layer as olayer
    from tp_cpu_ops import expected_rank_grads
    import tensor_transformer_layer_column_b200 as tl
    out = _spawn(_grid_worker, 4)
    refs = []
    for dp in (0, 1):
        w, p64, x, dy = _batch(dp)
        refs.append(olayer.layer_bwd(x, p64, dy, w.batch, w.heads, True, w.ln_eps))
    dims = tl.Dims.of(w.batch, w.seq, w.hidden, w.ffn, w.heads, w.head_dim, w.t, 1, w.ln_eps)
    for rank, grads, order in out:
        dp, tp = divmod(rank, 2)
        assert order == ["mlp", "attn", "ln1"]
        want0 = expected_rank_grads(refs[0], dims, tp)
        want1 = expected_rank_grads(refs[1], dims, tp)
        for k in want0:
            want = 0.5 * (want0[k] + want1[k])
            err = np.abs(grads[k] - want).max()
            assert err <= 1e-10 * max(1.0, np.abs(want).max()), f"d{k} rank {rank}: {err:.3e}"
        # The two replicas' batches differ, so the average is not either one's own gradient.
        assert np.abs(want0["w1"] - want1["w1"]).max() > 1e-3
