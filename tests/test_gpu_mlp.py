"""Parity of the CUDA MLP sublayer (tp_mlp_fwd / tp_mlp_bwd) with the fp64 oracle.

"How transformer layers actually decompose": W1 column-split with local GeLU,
W2 row-split with the partial outputs summed; the backward sums the input
gradients of the column-parallel product over the shards.
"""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import layout as olay
from oracle import mlp as omlp
from parity import check, f64
from synth import Workload, make_inputs, to_f64, workload
from tensor_transformer_layer_column_b200.sublayer import ShardedMLP

pytestmark = pytest.mark.gpu


def _run(w, inp, resid=None, backward=True):
    d = dims_of(w)
    g = dev(inp)
    m = ShardedMLP(d, g["w1"], g["b1"], g["w2"], g["b2"])
    o = m.forward(g["x"], resid=None if resid is None else resid.cuda())
    grads = m.backward(g["dy"]) if backward else None
    torch.cuda.synchronize()
    assert_no_device_error()
    return o, grads


def _ref(w, inp, resid=None, backward=True):
    x, w1, b1, w2, b2 = (to_f64(inp[k]) for k in ("x", "w1", "b1", "w2", "b2"))
    y, a, h = omlp.mlp_fwd(x, w1, b1, w2, b2, None if resid is None else to_f64(resid))
    g = omlp.mlp_bwd(x, w1, b1, w2, to_f64(inp["dy"])) if backward else None
    return y, a, h, g


def _compare(w, o, grads, y, a, h, g):
    t = w.t
    check("y", o["y"], y)
    check("a_save", o["a"], olay.shard_cols(a, t))
    check("h_save", o["h"], olay.shard_cols(h, t))
    if g is not None:
        check("dx", grads["dx"], g["dx"])
        check("dw1", grads["dw1"], olay.shard_cols(g["dw1"], t))
        check("dw2", grads["dw2"], olay.shard_rows(g["dw2"], t))
        check("db1", grads["db1"], g["db1"])
        check("db2", grads["db2"], g["db2"])


def test_mlp_fwd_workload_T128_D256_F1024_t2():
    require_gpu()
    w = workload("mlp_fwd_T128_D256_F1024_t2")
    inp = make_inputs(w, with_dy=True)
    o, grads = _run(w, inp)
    y, a, h, g = _ref(w, inp)
    _compare(w, o, grads, y, a, h, g)


# Shapes spanning several 128x256 tiles, ragged token counts (M tails),
# hidden/ffn widths that are not tile multiples (N and K tails) and every t.
SMALL = [
    (2, 100, 256, 2048, 2),
    (1, 333, 512, 4096, 8),
    (3, 50, 264, 1040, 2),
    (1, 7, 128, 512, 4),
    (2, 64, 256, 1024, 1),
    (1, 300, 1024, 2048, 8),
]


@pytest.mark.parametrize("batch,seq,D,F,t", SMALL)
@pytest.mark.parametrize("affine", [False, True])
def test_mlp_fwd_bwd_small(batch, seq, D, F, t, affine):
    require_gpu()
    w = Workload("mlp_test", "mlp_fwdbwd", batch=batch, seq=seq, hidden=D, ffn=F, t=t)
    inp = make_inputs(w, seed=3, random_affine=affine)
    resid = inp.get("resid")
    o, grads = _run(w, inp, resid=resid)
    y, a, h, g = _ref(w, inp, resid=resid)
    _compare(w, o, grads, y, a, h, g)


def test_mlp_bwd_residual_gradient_passes_through():
    require_gpu()
    w = Workload("mlp_test", "mlp_fwdbwd", batch=1, seq=130, hidden=256, ffn=1024, t=4)
    inp = make_inputs(w, seed=5)
    d = dims_of(w)
    g = dev(inp)
    m = ShardedMLP(d, g["w1"], g["b1"], g["w2"], g["b2"])
    m.forward(g["x"])
    gr = m.backward(g["dy"], dres=g["dy"])
    ref = omlp.mlp_bwd(*(to_f64(inp[k]) for k in ("x", "w1", "b1", "w2", "dy")))
    check("dx + dres", gr["dx"], ref["dx"] + to_f64(inp["dy"]))


def test_mlp_deterministic_run_to_run():
    require_gpu()
    w = Workload("mlp_test", "mlp_fwdbwd", batch=2, seq=256, hidden=512, ffn=2048, t=8)
    inp = make_inputs(w, seed=11, random_affine=True)
    o1, g1 = _run(w, inp)
    o2, g2 = _run(w, inp)
    for k in ("y", "a", "h"):
        assert torch.equal(o1[k], o2[k]), k
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_mlp_zero_tokens():
    require_gpu()
    w = Workload("mlp_test", "mlp_fwdbwd", batch=0, seq=16, hidden=256, ffn=1024, t=2)
    d = dims_of(w)
    rng = torch.Generator().manual_seed(0)
    w1 = torch.randn(256, 1024, generator=rng).to(torch.bfloat16).cuda()
    w2 = torch.randn(1024, 256, generator=rng).to(torch.bfloat16).cuda()
    m = ShardedMLP(d, w1, None, w2, None)
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    m.forward(x)
    grads = {"dx": torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"),
             "dw1": torch.full((2, 256, 512), 7.0, dtype=torch.bfloat16, device="cuda"),
             "dw2": torch.full((2, 512, 256), 7.0, dtype=torch.bfloat16, device="cuda"),
             "db1": torch.full((1024,), 7.0, dtype=torch.bfloat16, device="cuda"),
             "db2": torch.full((256,), 7.0, dtype=torch.bfloat16, device="cuda")}
    m.backward(x, out=grads)
    torch.cuda.synchronize()
    for k in ("dw1", "dw2", "db1", "db2"):
        assert torch.count_nonzero(grads[k]) == 0, k


def test_mlp_full_size_T8192_D3072_F12288_t8():
    """The 8.3B-width workload, every output and gradient against the full oracle."""
    require_gpu()
    w = workload("mlp_fwdbwd_T8192_D3072_F12288_t8")
    inp = make_inputs(w)
    o, grads = _run(w, inp)
    y, a, h, g = _ref(w, inp)
    _compare(w, o, grads, y, a, h, g)


def c4_sample_rows_cols(T, F, t):
    """Rows: every 16th token and the last row of every 128-row block (both
    sides of every tile edge of the 128- and 256-row tiles).  FFN columns:
    every 16th, plus the first and last column of every 256-wide tile of every
    shard (the column tiles restart at each shard's boundary)."""
    rows = set(range(0, T, 16)) | set(range(127, T, 128))
    ft = F // t
    cols = set(range(0, F, 16))
    for i in range(t):
        for n0 in range(0, ft, 256):
            cols |= {i * ft + n0, i * ft + min(n0 + 255, ft - 1)}
    return np.array(sorted(rows)), np.array(sorted(cols))


def test_c4_sample_covers_every_tile_edge():
    T, F, t = 8192, 28672, 8
    R, J = c4_sample_rows_cols(T, F, t)
    assert len(R) == 8192 // 16 + 64 and {0, 127, 128, 255, 256, T - 1} <= set(R)
    ft = F // t
    assert {0, 255, 256, ft - 1, ft, ft + 255, F - 1} <= set(J) and len(J) > F // 16


def test_mlp_full_size_T8192_D7168_F28672_t8_sampled():
    """The 30B FFN shape, checked on ~600 rows (y, dx, saved activations) and
    ~2000 ffn columns (dW1 columns, dW2 rows, db1) that include every tile edge:
    the MLP decomposes exactly over rows of x and over columns of W1 / rows of
    W2, so the oracle computes each sample from the same definition on a slice."""
    require_gpu()
    w = workload("mlp_fwdbwd_T8192_D7168_F28672_t8")
    inp = make_inputs(w)
    o, grads = _run(w, inp)
    T, D, F, t = w.tokens, w.hidden, w.ffn, w.t
    ft = F // t
    R, J = c4_sample_rows_cols(T, F, t)
    x, w1, b1, w2, b2, dy = (to_f64(inp[k]) for k in ("x", "w1", "b1", "w2", "b2", "dy"))
    y, a, h = omlp.mlp_fwd(x[R], w1, b1, w2, b2)
    check("y[rows]", f64(o["y"])[R], y)
    a_g = f64(o["a"]).transpose(1, 0, 2).reshape(T, F)
    h_g = f64(o["h"]).transpose(1, 0, 2).reshape(T, F)
    check("a_save[rows]", a_g[R], a)
    check("h_save[rows]", h_g[R], h)
    del a_g, h_g
    gr = omlp.mlp_bwd(x[R], w1, b1, w2, dy[R])
    check("dx[rows]", f64(grads["dx"])[R], gr["dx"])
    gc = omlp.mlp_bwd(x, w1[:, J], b1[J], w2[J, :], dy)
    dw1 = f64(grads["dw1"])
    dw1_j = np.stack([dw1[j // ft][:, j % ft] for j in J], axis=1)
    check("dw1[:, cols]", dw1_j, gc["dw1"])
    dw2 = f64(grads["dw2"]).reshape(F, D)
    check("dw2[cols, :]", dw2[J], gc["dw2"])
    check("db1[cols]", f64(grads["db1"])[J], gc["db1"])
    check("db2", grads["db2"], dy.sum(axis=0))
