"""Pins of the tensor-parallel identities the pages state (CPU only).

"How transformer layers actually decompose": the t row-parallel partials of
column-sharded GeLU(x W1_i) W2_i sum to the unsharded GeLU(x W1) W2; GeLU is
local to each shard because it is elementwise.  "The attention heads split":
head-sliced attention with a row-split output projection equals full
multi-head attention.  The explainer's "column comes first" takeaway is the
negative control: splitting W1 by rows would need a sum before GeLU.
"""
import json
import os

import numpy as np
import pytest

from oracle import attention, core, layout, mlp, sharded

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(99)


def _rel(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_mlp_sharding_identity_fwd_bwd(t):
    T, D, F_ = 6, 16, 64
    x = RNG.normal(size=(T, D))
    w1, b1 = RNG.normal(size=(D, F_)) * 0.3, RNG.normal(size=F_) * 0.1
    w2, b2 = RNG.normal(size=(F_, D)) * 0.3, RNG.normal(size=D) * 0.1
    dy = RNG.normal(size=(T, D))
    y, _, _ = mlp.mlp_fwd(x, w1, b1, w2, b2)
    assert _rel(sharded.mlp_fwd_sharded(x, w1, b1, w2, b2, t), y) < 1e-13
    g = mlp.mlp_bwd(x, w1, b1, w2, dy)
    gs = sharded.mlp_bwd_sharded(x, w1, b1, w2, dy, t)
    for k in g:
        assert _rel(gs[k], g[k]) < 1e-13, k


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_attention_head_slicing_identity_fwd_bwd(t):
    B, S, H, dh = 2, 5, 8, 3
    D = H * dh
    x = RNG.normal(size=(B * S, D))
    wqkv, bqkv = RNG.normal(size=(D, 3 * D)) * 0.4, RNG.normal(size=3 * D) * 0.1
    wout, bout = RNG.normal(size=(D, D)) * 0.4, RNG.normal(size=D) * 0.1
    dy = RNG.normal(size=(B * S, D))
    y, _ = attention.attn_fwd(x, wqkv, bqkv, wout, bout, B, H)
    assert _rel(sharded.attn_fwd_sharded(x, wqkv, bqkv, wout, bout, B, H, t), y) < 1e-13
    g = attention.attn_bwd(x, wqkv, bqkv, wout, dy, B, H)
    gs = sharded.attn_bwd_sharded(x, wqkv, bqkv, wout, dy, B, H, t)
    for k in gs:
        assert _rel(gs[k], g[k]) < 1e-13, k


def test_gelu_is_local_to_column_shards():
    x = RNG.normal(size=(7, 12))
    w1 = RNG.normal(size=(12, 32))
    a = x @ w1
    full = core.gelu(a)
    for i, blk in enumerate(layout.shard_cols(a, 4)):
        # Elementwise: the block of GeLU(A) is exactly GeLU of the block.
        np.testing.assert_array_equal(full[:, i * 8:(i + 1) * 8], core.gelu(blk))
    for i, w1_i in enumerate(layout.shard_cols(w1, 4)):
        np.testing.assert_allclose(a[:, i * 8:(i + 1) * 8], x @ w1_i, rtol=0, atol=1e-13)


def test_row_split_of_w1_is_not_local_negative_control():
    T, D, F_, t = 6, 16, 32, 2
    x = RNG.normal(size=(T, D))
    w1 = RNG.normal(size=(D, F_)) * 0.5
    w2 = RNG.normal(size=(F_, D)) * 0.5
    ref = core.gelu(x @ w1) @ w2
    dt = D // t
    # Wrong order: W1 split by rows needs the partial products summed BEFORE GeLU.
    wrong = sum(core.gelu(x[:, i * dt:(i + 1) * dt] @ w1[i * dt:(i + 1) * dt, :]) @ w2
                for i in range(t))
    assert _rel(wrong, ref) > 0.1
    right = core.gelu(sum(x[:, i * dt:(i + 1) * dt] @ w1[i * dt:(i + 1) * dt, :]
                          for i in range(t))) @ w2
    assert _rel(right, ref) < 1e-13


def test_bias_of_row_parallel_output_is_added_once():
    T, D, F_, t = 4, 8, 16, 4
    x = RNG.normal(size=(T, D))
    w1, b1 = RNG.normal(size=(D, F_)), RNG.normal(size=F_)
    w2, b2 = RNG.normal(size=(F_, D)), RNG.normal(size=D)
    y, _, _ = mlp.mlp_fwd(x, w1, b1, w2, b2)
    ys = sharded.mlp_fwd_sharded(x, w1, b1, w2, b2, t)
    np.testing.assert_allclose(ys, y, atol=1e-12)
    # Adding b2 once per shard would move every row by (t - 1) b2.
    wrong = ys + (t - 1) * b2
    assert np.abs(wrong - y).max() > 0.1 * np.abs(b2).max()


def test_two_way_split_shapes_from_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "two_way_split_shapes.json")))
    hidden = 8
    w1 = np.zeros((hidden, 4 * hidden))
    w2 = np.zeros((4 * hidden, hidden))
    s1 = layout.shard_cols(w1, g["t"])
    s2 = layout.shard_rows(w2, g["t"])
    assert s1.shape[1:] == tuple(v * hidden for v in g["w1_shard_shape_in_units_of_hidden"])
    assert s2.shape[1:] == tuple(v * hidden for v in g["w2_shard_shape_in_units_of_hidden"])
    x = np.zeros((3, hidden))
    assert (x @ s1[0]).shape[1] == g["intermediate_width_in_units_of_hidden"] * hidden
    assert ((x @ s1[0]) @ s2[0]).shape[1] == g["partial_output_width_in_units_of_hidden"] * hidden


def test_30b_ffn_weight_size_from_the_pages():
    from synth import workload
    g = json.load(open(os.path.join(GOLDEN, "ffn_30b_shapes.json")))
    w = workload("mlp_fwdbwd_T8192_D7168_F28672_t8")
    assert [w.hidden, w.ffn] == g["w1_shape"] and [w.ffn, w.hidden] == g["w2_shape"]
    nbytes = w.hidden * w.ffn * g["bytes_per_element"]
    assert nbytes == 411_041_792
    assert round(nbytes / 1e6) == g["approx_mb_per_matrix"]
    assert abs(2 * nbytes / 1e6 - g["approx_mb_per_layer"]) < 1.0


def _layer_params(D, F_):
    p = {"ln1_g": 1 + 0.1 * RNG.normal(size=D), "ln1_b": 0.1 * RNG.normal(size=D),
         "wqkv": 0.4 * RNG.normal(size=(D, 3 * D)), "bqkv": 0.1 * RNG.normal(size=3 * D),
         "wout": 0.4 * RNG.normal(size=(D, D)), "bout": 0.1 * RNG.normal(size=D),
         "ln2_g": 1 + 0.1 * RNG.normal(size=D), "ln2_b": 0.1 * RNG.normal(size=D),
         "w1": 0.3 * RNG.normal(size=(D, F_)), "b1": 0.1 * RNG.normal(size=F_),
         "w2": 0.3 * RNG.normal(size=(F_, D)), "b2": 0.1 * RNG.normal(size=D)}
    return p


@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("placement", ["pre", "post"])
def test_layer_built_from_sharded_sublayers(t, placement):
    """Both layer placements composed from the sharded sublayers (each with its
    own shard sums) equal the unsharded layers, forward and backward."""
    from oracle import layer as olayer
    B, S, H, dh, F_ = 2, 5, 8, 3, 64
    D = H * dh
    p = _layer_params(D, F_)
    x = RNG.normal(size=(B * S, D))
    dy = RNG.normal(size=(B * S, D))

    def attn_s(u):
        return sharded.attn_fwd_sharded(u, p["wqkv"], p["bqkv"], p["wout"], p["bout"], B, H, t)

    def mlp_s(u):
        return sharded.mlp_fwd_sharded(u, p["w1"], p["b1"], p["w2"], p["b2"], t)

    ln = core.layernorm_fwd
    if placement == "pre":
        u1, m1, r1 = ln(x, p["ln1_g"], p["ln1_b"], 1e-5)
        h = x + attn_s(u1)
        u2, m2, r2 = ln(h, p["ln2_g"], p["ln2_b"], 1e-5)
        y = h + mlp_s(u2)
        yr, _ = olayer.layer_fwd(x, p, B, H)
        gm = sharded.mlp_bwd_sharded(u2, p["w1"], p["b1"], p["w2"], dy, t)
        du2, _, _ = core.layernorm_bwd(gm["dx"], h, p["ln2_g"], m2, r2)
        dh = dy + du2
        ga = sharded.attn_bwd_sharded(u1, p["wqkv"], p["bqkv"], p["wout"], dh, B, H, t)
        du1, _, _ = core.layernorm_bwd(ga["dx"], x, p["ln1_g"], m1, r1)
        dx = dh + du1
        gr = olayer.layer_bwd(x, p, dy, B, H)
    else:
        z1 = x + attn_s(x)
        h, m1, r1 = ln(z1, p["ln1_g"], p["ln1_b"], 1e-5)
        z2 = h + mlp_s(h)
        y, m2, r2 = ln(z2, p["ln2_g"], p["ln2_b"], 1e-5)
        yr, _ = olayer.postln_layer_fwd(x, p, B, H)
        dz2, _, _ = core.layernorm_bwd(dy, z2, p["ln2_g"], m2, r2)
        gm = sharded.mlp_bwd_sharded(h, p["w1"], p["b1"], p["w2"], dz2, t)
        dh = dz2 + gm["dx"]
        dz1, _, _ = core.layernorm_bwd(dh, z1, p["ln1_g"], m1, r1)
        ga = sharded.attn_bwd_sharded(x, p["wqkv"], p["bqkv"], p["wout"], dz1, B, H, t)
        dx = dz1 + ga["dx"]
        gr = olayer.postln_layer_bwd(x, p, dy, B, H)
    assert _rel(y, yr) < 1e-12
    assert _rel(dx, gr["dx"]) < 1e-12
    for k, v in (("dw1", gm["dw1"]), ("dw2", gm["dw2"]), ("dwqkv", ga["dwqkv"]),
                 ("dwout", ga["dwout"]), ("db1", gm["db1"]), ("dbqkv", ga["dbqkv"])):
        assert _rel(v, gr[k]) < 1e-12, k
