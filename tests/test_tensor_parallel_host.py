"""Host logic of the one-shard-per-GPU layer (CPU only).

tensor_parallel.RankLayer / layer_forward / layer_backward sequence, for each
rank, the work between the pages' exchange points ("One Idea, Two
Insertions": one all-reduce per sublayer in the forward pass and one in the
backward pass).  Here the per-rank arithmetic is the oracle's fp64 primitives
(tests/tp_cpu_ops.py), so these tests pin the host logic alone: the phase
order, that exactly the row-parallel partials and the column-parallel input
gradients are summed, that the row-parallel biases enter once, and where each
gradient lands -- against the unsharded oracle layer, to fp64 rounding.

Two exchanges: LocalSum (one process drives all t ranks) and AllReduce over
world-size 2 and 4 gloo process groups (one rank per process).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import layer as olayer
from synth import Workload, make_inputs, to_f64

PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2",
          "b2")


def _case(t):
    w = Workload("tp_host", "layer_fwdbwd", batch=2, seq=12, hidden=32, ffn=64, heads=8,
                 head_dim=4, t=t)
    inp = make_inputs(w, seed=5, random_affine=True)
    p64 = {k: to_f64(inp[k]) for k in PARAMS}
    return w, p64, to_f64(inp["x"]), to_f64(inp["dy"])


def _dims(w):
    import tensor_transformer_layer_column_b200 as tl
    return tl.Dims.of(w.batch, w.seq, w.hidden, w.ffn, w.heads, w.head_dim, w.t, 1, w.ln_eps)


def _reference(w, p64, x, dy):
    y, _ = olayer.layer_fwd(x, p64, w.batch, w.heads, True, w.ln_eps)
    g = olayer.layer_bwd(x, p64, dy, w.batch, w.heads, True, w.ln_eps)
    return y, g


def _close(name, got, want):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - want).max()
    assert err <= 1e-10 * max(1.0, np.abs(want).max()), f"{name}: max err {err:.3e}"


def _run_ranks(w, p64, x, dy, ranks_idx, exchange):
    from tensor_transformer_layer_column_b200.tensor_parallel import (RankLayer, layer_backward,
                                                                      layer_forward)
    from tp_cpu_ops import OracleRankOps, rank_params
    dims = _dims(w)
    ranks = [RankLayer(dims, i, rank_params(p64, dims, i), OracleRankOps(dims)) for i in ranks_idx]
    xt, dyt = torch.from_numpy(x), torch.from_numpy(dy)
    ready = []
    ys = layer_forward(ranks, xt, exchange)
    n_fwd = exchange.count
    dxs = layer_backward(ranks, dyt, exchange, on_grads_ready=ready.append)
    return ranks, ys, dxs, n_fwd, exchange.count - n_fwd, ready


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_local_sum_of_all_ranks_equals_the_unsharded_layer(t):
    from tensor_transformer_layer_column_b200.tensor_parallel import LocalSum
    from tp_cpu_ops import expected_rank_grads
    w, p64, x, dy = _case(t)
    y_ref, g_ref = _reference(w, p64, x, dy)
    ranks, ys, dxs, n_fwd, n_bwd, ready = _run_ranks(w, p64, x, dy, range(t), LocalSum())
    assert (n_fwd, n_bwd) == (2, 2)          # one exchange per sublayer per direction
    assert ready == ["mlp", "attn", "ln1"]
    dims = _dims(w)
    for r, y, dx in zip(ranks, ys, dxs):
        _close(f"y (rank {r.rank})", y.numpy(), y_ref)
        _close(f"dx (rank {r.rank})", dx.numpy(), g_ref["dx"])
        want = expected_rank_grads(g_ref, dims, r.rank)
        for k, v in want.items():
            _close(f"d{k} (rank {r.rank})", r.grads[k].numpy(), v)


def test_a_missing_rank_partial_is_detected():
    """Negative control: dropping one rank's partial from the sum changes y,
    so the comparison above would catch an exchange that loses a shard."""
    from tensor_transformer_layer_column_b200.tensor_parallel import LocalSum

    class DropLast(LocalSum):
        def __call__(self, partials):
            self.count += 1
            return list(partials)[:-1]

    w, p64, x, dy = _case(4)
    y_ref, _ = _reference(w, p64, x, dy)
    _, ys, _, _, _, _ = _run_ranks(w, p64, x, dy, range(4), DropLast())
    assert np.abs(ys[0].numpy() - y_ref).max() > 1e-3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, os.path.dirname(here))
    sys.path.insert(0, here)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from tensor_transformer_layer_column_b200.tensor_parallel import AllReduce
        w, p64, x, dy = _case(world)
        ranks, ys, dxs, n_fwd, n_bwd, ready = _run_ranks(w, p64, x, dy, [rank], AllReduce())
        q.put((rank, ys[0].numpy(), dxs[0].numpy(),
               {k: v.numpy() for k, v in ranks[0].grads.items()}, n_fwd, n_bwd, ready))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_allreduce_over_gloo_ranks_equals_the_unsharded_layer(world):
    from tp_cpu_ops import expected_rank_grads
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, p64, x, dy = _case(world)
    y_ref, g_ref = _reference(w, p64, x, dy)
    dims = _dims(w)
    for rank, y, dx, grads, n_fwd, n_bwd, ready in sorted(out, key=lambda o: o[0]):
        assert (n_fwd, n_bwd) == (2, 2)
        assert ready == ["mlp", "attn", "ln1"]
        _close(f"y (rank {rank})", y, y_ref)
        _close(f"dx (rank {rank})", dx, g_ref["dx"])
        for k, v in expected_rank_grads(g_ref, dims, rank).items():
            _close(f"d{k} (rank {rank})", grads[k], v)
