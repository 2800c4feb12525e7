"""Parity of the one-shard-per-GPU entry points with the fp64 oracle.

The pages' deployment ("One Idea, Two Insertions"; "How transformer layers
actually decompose"): rank i runs shard i between the exchange points and
contributes an fp32 partial; the partials are summed and tp_rowpar_finish adds
the row-parallel bias once and the residual.  With one GPU here, the t ranks
run one after another on it (nothing waits on anything else: the exchange is
the finish kernel reading all t partials), and every output and gradient is
compared with the unsharded oracle, cut to each rank's shard.
"""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import attention as oatt
from oracle import layer as olayer
from oracle import layout as olay
from oracle import mlp as omlp
from parity import check
from synth import Workload, make_inputs, to_f64
from tensor_transformer_layer_column_b200.sublayer import pack_cols, pack_qkv, pack_rows
from tensor_transformer_layer_column_b200.tensor_parallel import (LibraryRankOps, LocalSum,
                                                                  RankLayer, layer_backward,
                                                                  layer_forward,
                                                                  shard_layer_params)

pytestmark = pytest.mark.gpu
BF, F16, F32 = torch.bfloat16, torch.float16, torch.float32
PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2",
          "b2")


def _empty(shape, dtype=BF):
    return torch.empty(shape, dtype=dtype, device="cuda")


def _ws(op, d):
    n = tl.rank_workspace_size(op, d)
    return torch.empty(max(n, 1), dtype=torch.uint8, device="cuda") if n else None


@pytest.mark.parametrize("T,D,F,t", [(100, 256, 1024, 1), (100, 256, 1024, 2), (300, 512, 2048, 4),
                                     (257, 256, 2048, 8)])
def test_rank_mlp_forward_backward(T, D, F, t):
    require_gpu()
    w = Workload("rank_mlp", "mlp_fwdbwd", batch=1, seq=T, hidden=D, ffn=F, t=t)
    inp = make_inputs(w, seed=21, random_affine=True)
    g = dev(inp)
    d = dims_of(w)
    Ft = F // t
    w1s, w2s = pack_cols(g["w1"], t), pack_rows(g["w2"], t)
    b1s = g["b1"].reshape(t, Ft)
    a = [_empty((T, Ft)) for _ in range(t)]
    h = [_empty((T, Ft)) for _ in range(t)]
    parts = [_empty((T, D), F32) for _ in range(t)]
    for i in range(t):
        tl.mlp_fwd_rank(d, g["x"], w1s[i], b1s[i], w2s[i], a[i], h[i], parts[i])
    y = _empty((T, D))
    tl.rowpar_finish(parts, g["b2"], g["resid"], T, D, y)
    dparts = [_empty((T, D), F32) for _ in range(t)]
    dw1 = [_empty((D, Ft)) for _ in range(t)]
    dw2 = [_empty((Ft, D)) for _ in range(t)]
    db1 = [_empty((Ft,)) for _ in range(t)]
    db2 = _empty((D,))
    ws = _ws(tl.RANK_MLP_BWD, d)
    for i in range(t):
        tl.mlp_bwd_rank(d, g["x"], w1s[i], w2s[i], a[i], h[i], g["dy"], dw1[i], dw2[i], db1[i],
                        db2 if i == 0 else None, dparts[i], ws)
    dx = _empty((T, D))
    tl.rowpar_finish(dparts, None, g["resid"], T, D, dx)
    torch.cuda.synchronize()
    assert_no_device_error()

    x, w1, b1, w2, b2, r, dy = (to_f64(inp[k]) for k in ("x", "w1", "b1", "w2", "b2", "resid", "dy"))
    yr, ar, hr = omlp.mlp_fwd(x, w1, b1, w2, b2, resid=r)
    check("y", y, yr)
    gr = omlp.mlp_bwd(x, w1, b1, w2, dy)
    check("dx", dx, gr["dx"] + r)
    for i in range(t):
        cols = slice(i * Ft, (i + 1) * Ft)
        check(f"a[{i}]", a[i], ar[:, cols])
        check(f"h[{i}]", h[i], hr[:, cols])
        check(f"dw1[{i}]", dw1[i], gr["dw1"][:, cols])
        check(f"dw2[{i}]", dw2[i], gr["dw2"][cols, :])
        check(f"db1[{i}]", db1[i], gr["db1"][cols])
    check("db2", db2, gr["db2"])


@pytest.mark.parametrize("B,S,H,dh,t,causal", [(2, 100, 4, 64, 2, True), (1, 257, 8, 128, 8, True),
                                               (2, 96, 4, 128, 4, False), (1, 64, 2, 64, 1, True)])
def test_rank_attention_forward_backward(B, S, H, dh, t, causal):
    require_gpu()
    D = H * dh
    w = Workload("rank_attn", "attn_fwdbwd", batch=B, seq=S, hidden=D, heads=H, head_dim=dh, t=t,
                 causal=causal)
    inp = make_inputs(w, seed=23, random_affine=True)
    g = dev(inp)
    d = dims_of(w)
    T, Dt, Hl = B * S, D // t, H // t
    wq, wo = pack_qkv(g["wqkv"], H, t), pack_rows(g["wout"], t)
    bq = pack_qkv(g["bqkv"], H, t)
    qkv = [_empty((T, 3 * Dt), F16) for _ in range(t)]
    o = [_empty((T, Dt)) for _ in range(t)]
    lse = [_empty((B, Hl, S), F32) for _ in range(t)]
    parts = [_empty((T, D), F32) for _ in range(t)]
    wsf = _ws(tl.RANK_ATTN_FWD, d)
    for i in range(t):
        tl.attn_fwd_rank(d, g["x"], None, wq[i], bq[i], wo[i], qkv[i], o[i], lse[i], parts[i], wsf)
    y = _empty((T, D))
    tl.rowpar_finish(parts, g["bout"], g["resid"], T, D, y)
    wsb = _ws(tl.RANK_ATTN_BWD, d)
    dparts = [_empty((T, D), F32) for _ in range(t)]
    dwq = [_empty((D, 3 * Dt)) for _ in range(t)]
    dbq = [_empty((3 * Dt,)) for _ in range(t)]
    dwo = [_empty((Dt, D)) for _ in range(t)]
    dbo = _empty((D,))
    for i in range(t):
        tl.attn_bwd_rank(d, g["x"], None, wq[i], wo[i], qkv[i], o[i], lse[i], g["dy"], dwq[i],
                         dbq[i], dwo[i], dbo if i == 0 else None, dparts[i], wsb)
    dx = _empty((T, D))
    tl.rowpar_finish(dparts, None, None, T, D, dx)
    torch.cuda.synchronize()
    assert_no_device_error()

    x, wqkv, bqkv, wout, bout, r, dy = (to_f64(inp[k]) for k in
                                        ("x", "wqkv", "bqkv", "wout", "bout", "resid", "dy"))
    yr, sv = oatt.attn_fwd(x, wqkv, bqkv, wout, bout, B, H, causal, resid=r)
    check("y", y, yr)
    gr = oatt.attn_bwd(x, wqkv, bqkv, wout, dy, B, H, causal)
    check("dx", dx, gr["dx"])
    qkv_r = olay.shard_qkv(sv["qkv"], t)
    o_r = olay.shard_cols(sv["o"], t)
    dwq_r = olay.shard_qkv(gr["dwqkv"], t)
    dbq_r = olay.shard_qkv(gr["dbqkv"][None, :], t)
    dwo_r = olay.shard_rows(gr["dwout"], t)
    for i in range(t):
        check(f"qkv[{i}]", qkv[i], qkv_r[i])
        check(f"o[{i}]", o[i], o_r[i])
        check(f"lse[{i}]", lse[i], sv["lse"][:, i * Hl:(i + 1) * Hl, :])
        check(f"dwqkv[{i}]", dwq[i], dwq_r[i])
        check(f"dbqkv[{i}]", dbq[i], dbq_r[i][0])
        check(f"dwout[{i}]", dwo[i], dwo_r[i])
    check("dbout", dbo, gr["dbout"])


def test_rowpar_finish_sums_in_rank_order_and_adds_bias_once():
    """out = bf16(p0 + p1 + p2 + bias + resid), bit for bit against the same
    fp32 additions in the same order, rounded to bf16 once."""
    require_gpu()
    gen = torch.Generator().manual_seed(3)
    rows, cols = 37, 96
    parts = [torch.randn(rows, cols, generator=gen) * 10 for _ in range(3)]
    bias = torch.randn(cols, generator=gen).to(BF)
    resid = torch.randn(rows, cols, generator=gen).to(BF)
    out, out32 = _empty((rows, cols)), _empty((rows, cols), F32)
    tl.rowpar_finish([p.cuda() for p in parts], bias.cuda(), resid.cuda(), rows, cols, out, out32)
    torch.cuda.synchronize()
    want = ((parts[0] + parts[1]) + parts[2]) + bias.float() + resid.float()
    assert torch.equal(out32.cpu(), want)
    assert torch.equal(out.cpu(), want.to(BF))


def _layer_compare(w, inp, ref=None):
    d = dims_of(w)
    g = dev(inp)
    t = w.t
    ranks = [RankLayer(d, i, shard_layer_params({k: g[k] for k in PARAMS}, d, i),
                       LibraryRankOps(d, "cuda")) for i in range(t)]
    ex = LocalSum()
    ys = layer_forward(ranks, g["x"], ex)
    dxs = layer_backward(ranks, g["dy"], ex)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert ex.count == 4
    if ref is None:
        p = {k: to_f64(inp[k]) for k in PARAMS}
        x = to_f64(inp["x"])
        yr, _ = olayer.layer_fwd(x, p, w.batch, w.heads, w.causal, w.ln_eps)
        gr = olayer.layer_bwd(x, p, to_f64(inp["dy"]), w.batch, w.heads, w.causal, w.ln_eps)
    else:
        yr, gr = ref
    for i in (0, t - 1):       # every rank computes the same y and dx
        assert torch.equal(ys[i], ys[0]) and torch.equal(dxs[i], dxs[0])
    check("y", ys[0], yr)
    check("dx", dxs[0], gr["dx"])
    dwq, dbq = olay.shard_qkv(gr["dwqkv"], t), olay.shard_qkv(gr["dbqkv"][None, :], t)
    dwo, dw1, dw2 = (olay.shard_rows(gr["dwout"], t), olay.shard_cols(gr["dw1"], t),
                     olay.shard_rows(gr["dw2"], t))
    db1 = gr["db1"].reshape(t, -1)
    for r in ranks:
        i, gg = r.rank, r.grads
        check(f"dwqkv[{i}]", gg["wqkv"], dwq[i])
        check(f"dbqkv[{i}]", gg["bqkv"], dbq[i][0])
        check(f"dwout[{i}]", gg["wout"], dwo[i])
        check(f"dw1[{i}]", gg["w1"], dw1[i])
        check(f"db1[{i}]", gg["b1"], db1[i])
        check(f"dw2[{i}]", gg["w2"], dw2[i])
    for k, name in (("bout", "dbout"), ("b2", "db2"), ("ln1_g", "dln1_g"), ("ln1_b", "dln1_b"),
                    ("ln2_g", "dln2_g"), ("ln2_b", "dln2_b")):
        check(name, ranks[0].grads[k], gr[name])


@pytest.mark.parametrize("B,S,H,dh,F,t", [(2, 128, 4, 64, 1024, 2), (1, 200, 8, 64, 2048, 8),
                                          (2, 96, 4, 128, 1024, 4)])
def test_rank_layer_all_ranks_on_one_gpu(B, S, H, dh, F, t):
    require_gpu()
    w = Workload("rank_layer", "layer_fwdbwd", batch=B, seq=S, hidden=H * dh, ffn=F, heads=H,
                 head_dim=dh, t=t)
    _layer_compare(w, make_inputs(w, seed=29, random_affine=True))


def test_rank_layer_full_size_B4_S2048_D4096_H32_F16384_t8():
    """The pre-LN layer at its full size, eight ranks one after another on one
    GPU, every output and every rank's gradients against the full oracle."""
    require_gpu()
    from full_size_reference import pre_ln_layer
    w, inp, yr, _, gr = pre_ln_layer()
    _layer_compare(w, inp, ref=(yr, gr))
