"""Pins of the oracle's MLP, attention and pre-LN layer (CPU only).

Each sublayer is checked against (a) brute-force scalar loops on tiny shapes,
(b) central finite differences for every gradient, (c) an fp64 torch autograd
composition of library routines, and (d) closed-form special cases.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import brute_force as bf
from oracle import attention, layer, mlp

RNG = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return RNG.normal(size=shape) * scale


# ---------------------------------------------------------------- MLP

def _mlp_case(T=5, D=6, F_=12):
    return dict(x=_rand(T, D), w1=_rand(D, F_, scale=0.5), b1=_rand(F_, scale=0.3),
                w2=_rand(F_, D, scale=0.5), b2=_rand(D, scale=0.3))


def test_mlp_fwd_brute_force():
    c = _mlp_case()
    y, a, h = mlp.mlp_fwd(**c)
    yb = np.array(bf.mlp_fwd(c["x"].tolist(), c["w1"].tolist(), c["b1"].tolist(),
                             c["w2"].tolist(), c["b2"].tolist()))
    np.testing.assert_allclose(y, yb, rtol=0, atol=1e-12)


def test_mlp_residual_and_linearity_in_w2():
    c = _mlp_case()
    r = _rand(5, 6)
    y0, _, _ = mlp.mlp_fwd(**c)
    yr, _, _ = mlp.mlp_fwd(**c, resid=r)
    np.testing.assert_allclose(yr - y0, r, atol=1e-13)
    c2 = dict(c, w2=2.5 * c["w2"])
    y2, _, _ = mlp.mlp_fwd(**c2)
    np.testing.assert_allclose(y2 - c["b2"], 2.5 * (y0 - c["b2"]), atol=1e-12)


def test_mlp_bwd_finite_difference():
    c = _mlp_case(T=3, D=4, F_=8)
    dy = _rand(3, 4)
    g = mlp.mlp_bwd(c["x"], c["w1"], c["b1"], c["w2"], dy)

    def J(cc):
        return (mlp.mlp_fwd(**cc)[0] * dy).sum()

    h = 1e-6
    for name, gname in (("x", "dx"), ("w1", "dw1"), ("b1", "db1"), ("w2", "dw2"), ("b2", "db2")):
        fd = np.zeros_like(c[name])
        for idx in np.ndindex(c[name].shape):
            cp = {k: v.copy() for k, v in c.items()}
            cm = {k: v.copy() for k, v in c.items()}
            cp[name][idx] += h
            cm[name][idx] -= h
            fd[idx] = (J(cp) - J(cm)) / (2 * h)
        np.testing.assert_allclose(g[gname], fd, rtol=0, atol=1e-7, err_msg=gname)


def test_mlp_matches_torch_autograd():
    c = _mlp_case(T=7, D=16, F_=64)
    dy = _rand(7, 16)
    tc = {k: torch.tensor(v, requires_grad=True) for k, v in c.items()}
    y = F.gelu(tc["x"] @ tc["w1"] + tc["b1"], approximate="tanh") @ tc["w2"] + tc["b2"]
    y.backward(torch.tensor(dy))
    np.testing.assert_allclose(mlp.mlp_fwd(**c)[0], y.detach().numpy(), atol=1e-12)
    g = mlp.mlp_bwd(c["x"], c["w1"], c["b1"], c["w2"], dy)
    for name in ("x", "w1", "b1", "w2", "b2"):
        np.testing.assert_allclose(g["d" + name], tc[name].grad.numpy(), atol=1e-11)


# ---------------------------------------------------------------- attention

def _attn_case(B=2, S=4, H=2, dh=3):
    D = H * dh
    return dict(x=_rand(B * S, D), wqkv=_rand(D, 3 * D, scale=0.6), bqkv=_rand(3 * D, scale=0.3),
                wout=_rand(D, D, scale=0.5), bout=_rand(D, scale=0.3)), B, H


@pytest.mark.parametrize("causal", [True, False])
def test_attention_fwd_brute_force(causal):
    c, B, H = _attn_case()
    y, _ = attention.attn_fwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], c["bout"], B, H, causal)
    yb = np.array(bf.attention_fwd(c["x"].tolist(), c["wqkv"].tolist(), c["bqkv"].tolist(),
                                   c["wout"].tolist(), c["bout"].tolist(), B, H, causal))
    np.testing.assert_allclose(y, yb, rtol=0, atol=1e-12)


def test_attention_first_query_row_is_v0_and_seq1():
    c, B, H = _attn_case(B=3, S=5, H=2, dh=4)
    D = 8
    _, sv = attention.attn_fwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], c["bout"], B, H)
    v = sv["qkv"][:, 2 * D:]
    for b in range(B):
        np.testing.assert_allclose(sv["o"][b * 5], v[b * 5], atol=1e-14)
    # S = 1: every output row is its own v.
    c1, _, _ = _attn_case(B=4, S=1, H=2, dh=4)
    _, s1 = attention.attn_fwd(c1["x"], c1["wqkv"], c1["bqkv"], c1["wout"], c1["bout"], 4, 2)
    np.testing.assert_allclose(s1["o"], s1["qkv"][:, 2 * D:], atol=1e-14)


def test_attention_zero_keys_give_running_mean_of_v():
    c, B, H = _attn_case(B=2, S=6, H=2, dh=4)
    D = 8
    c["wqkv"][:, D:2 * D] = 0.0
    c["bqkv"][D:2 * D] = 0.0
    _, sv = attention.attn_fwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], c["bout"], B, H)
    v = sv["qkv"][:, 2 * D:]
    for b in range(B):
        for s in range(6):
            np.testing.assert_allclose(sv["o"][b * 6 + s], v[b * 6:b * 6 + s + 1].mean(axis=0),
                                       atol=1e-13)
    # lse of uniform scores over s+1 keys is log(s+1).
    np.testing.assert_allclose(sv["lse"][0, 0], np.log(np.arange(1, 7)), atol=1e-13)


def test_attention_core_matches_torch_sdpa():
    rng = np.random.default_rng(5)
    q, k, v = (rng.normal(size=(2, 3, 7, 5)) for _ in range(3))
    o, lse = attention.attn_core_fwd(q, k, v, causal=True)
    ref = F.scaled_dot_product_attention(torch.tensor(q), torch.tensor(k), torch.tensor(v),
                                         is_causal=True)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-13)
    s = torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) / np.sqrt(5)
    s = s.masked_fill(~torch.ones(7, 7, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-13)


def test_attention_bwd_finite_difference():
    c, B, H = _attn_case(B=2, S=3, H=2, dh=2)
    dy = _rand(6, 4)
    g = attention.attn_bwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], dy, B, H)

    def J(cc):
        return (attention.attn_fwd(cc["x"], cc["wqkv"], cc["bqkv"], cc["wout"], cc["bout"], B,
                                   H)[0] * dy).sum()

    h = 1e-6
    for name, gname in (("x", "dx"), ("wqkv", "dwqkv"), ("bqkv", "dbqkv"),
                        ("wout", "dwout"), ("bout", "dbout")):
        fd = np.zeros_like(c[name])
        for idx in np.ndindex(c[name].shape):
            cp = {k: v.copy() for k, v in c.items()}
            cm = {k: v.copy() for k, v in c.items()}
            cp[name][idx] += h
            cm[name][idx] -= h
            fd[idx] = (J(cp) - J(cm)) / (2 * h)
        np.testing.assert_allclose(g[gname], fd, rtol=0, atol=1e-7, err_msg=gname)


def _torch_attn(x, wqkv, bqkv, wout, bout, B, H):
    T, D = x.shape
    S = T // B
    qkv = x @ wqkv + bqkv
    q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(B, S, H, D // H).transpose(1, 2) for i in range(3))
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    return o.transpose(1, 2).reshape(T, D) @ wout + bout


def test_attention_matches_torch_autograd():
    c, B, H = _attn_case(B=2, S=9, H=4, dh=4)
    dy = _rand(18, 16)
    tc = {k: torch.tensor(v, requires_grad=True) for k, v in c.items()}
    y = _torch_attn(tc["x"], tc["wqkv"], tc["bqkv"], tc["wout"], tc["bout"], B, H)
    y.backward(torch.tensor(dy))
    y0, _ = attention.attn_fwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], c["bout"], B, H)
    np.testing.assert_allclose(y0, y.detach().numpy(), atol=1e-12)
    g = attention.attn_bwd(c["x"], c["wqkv"], c["bqkv"], c["wout"], dy, B, H)
    for name in ("x", "wqkv", "bqkv", "wout", "bout"):
        np.testing.assert_allclose(g["d" + name], tc[name].grad.numpy(), atol=1e-11)


# ---------------------------------------------------------------- pre-LN layer

def _layer_case(B=2, S=3, H=2, dh=2, F_=16):
    D = H * dh
    p = dict(ln1_g=1 + _rand(D, scale=0.2), ln1_b=_rand(D, scale=0.2),
             wqkv=_rand(D, 3 * D, scale=0.6), bqkv=_rand(3 * D, scale=0.2),
             wout=_rand(D, D, scale=0.5), bout=_rand(D, scale=0.2),
             ln2_g=1 + _rand(D, scale=0.2), ln2_b=_rand(D, scale=0.2),
             w1=_rand(D, F_, scale=0.5), b1=_rand(F_, scale=0.2),
             w2=_rand(F_, D, scale=0.5), b2=_rand(D, scale=0.2))
    return _rand(B * S, D), p, B, H


def test_layer_structure_is_pre_ln():
    x, p, B, H = _layer_case()
    y, sv = layer.layer_fwd(x, p, B, H)
    # y - h must equal MLP(LN2(h)) and h - x must equal Attn(LN1(x)).
    from oracle import core
    u1, _, _ = core.layernorm_fwd(x, p["ln1_g"], p["ln1_b"])
    a, _ = attention.attn_fwd(u1, p["wqkv"], p["bqkv"], p["wout"], p["bout"], B, H)
    np.testing.assert_allclose(sv["h"] - x, a, atol=1e-13)
    u2, _, _ = core.layernorm_fwd(sv["h"], p["ln2_g"], p["ln2_b"])
    m, _, _ = mlp.mlp_fwd(u2, p["w1"], p["b1"], p["w2"], p["b2"])
    np.testing.assert_allclose(y - sv["h"], m, atol=1e-13)


def test_layer_bwd_finite_difference():
    x, p, B, H = _layer_case()
    dy = _rand(*x.shape)
    g = layer.layer_bwd(x, p, dy, B, H)

    def J(xx, pp):
        return (layer.layer_fwd(xx, pp, B, H)[0] * dy).sum()

    h = 1e-6
    fd = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd[idx] = (J(xp, p) - J(xm, p)) / (2 * h)
    np.testing.assert_allclose(g["dx"], fd, rtol=0, atol=1e-7)
    for name in p:
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(p[name].shape):
            pp = {k: v.copy() for k, v in p.items()}
            pm = {k: v.copy() for k, v in p.items()}
            pp[name][idx] += h
            pm[name][idx] -= h
            fd[idx] = (J(x, pp) - J(x, pm)) / (2 * h)
        np.testing.assert_allclose(g["d" + name], fd, rtol=0, atol=1e-7, err_msg=name)


def test_layer_matches_torch_autograd():
    x, p, B, H = _layer_case(B=2, S=5, H=4, dh=4, F_=64)
    D = x.shape[1]
    dy = _rand(*x.shape)
    tx = torch.tensor(x, requires_grad=True)
    tp = {k: torch.tensor(v, requires_grad=True) for k, v in p.items()}
    u1 = F.layer_norm(tx, (D,), tp["ln1_g"], tp["ln1_b"], eps=1e-5)
    h = tx + _torch_attn(u1, tp["wqkv"], tp["bqkv"], tp["wout"], tp["bout"], B, H)
    u2 = F.layer_norm(h, (D,), tp["ln2_g"], tp["ln2_b"], eps=1e-5)
    y = h + F.gelu(u2 @ tp["w1"] + tp["b1"], approximate="tanh") @ tp["w2"] + tp["b2"]
    y.backward(torch.tensor(dy))
    y0, _ = layer.layer_fwd(x, p, B, H)
    np.testing.assert_allclose(y0, y.detach().numpy(), atol=1e-12)
    g = layer.layer_bwd(x, p, dy, B, H)
    np.testing.assert_allclose(g["dx"], tx.grad.numpy(), atol=1e-10)
    for name in p:
        np.testing.assert_allclose(g["d" + name], tp[name].grad.numpy(), atol=1e-10,
                                   err_msg=name)


# ---------------------------------------------------------------- post-LN layer

def test_postln_layer_structure():
    x, p, B, H = _layer_case()
    y, sv = layer.postln_layer_fwd(x, p, B, H)
    from oracle import core
    a, _ = attention.attn_fwd(x, p["wqkv"], p["bqkv"], p["wout"], p["bout"], B, H)
    np.testing.assert_allclose(sv["z1"], x + a, atol=1e-13)
    h, _, _ = core.layernorm_fwd(x + a, p["ln1_g"], p["ln1_b"])
    np.testing.assert_allclose(sv["h"], h, atol=1e-13)
    m, _, _ = mlp.mlp_fwd(h, p["w1"], p["b1"], p["w2"], p["b2"])
    yy, _, _ = core.layernorm_fwd(h + m, p["ln2_g"], p["ln2_b"])
    np.testing.assert_allclose(y, yy, atol=1e-13)
    # With beta = 0 and gamma = 1 every output row is normalised: mean 0, variance ~ 1.
    p1 = dict(p, ln2_g=np.ones_like(p["ln2_g"]), ln2_b=np.zeros_like(p["ln2_b"]))
    y1, _ = layer.postln_layer_fwd(x, p1, B, H)
    np.testing.assert_allclose(y1.mean(axis=1), 0, atol=1e-12)


def test_postln_layer_bwd_finite_difference():
    x, p, B, H = _layer_case()
    dy = _rand(*x.shape)
    g = layer.postln_layer_bwd(x, p, dy, B, H)

    def J(xx, pp):
        return (layer.postln_layer_fwd(xx, pp, B, H)[0] * dy).sum()

    h = 1e-6
    fd = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd[idx] = (J(xp, p) - J(xm, p)) / (2 * h)
    np.testing.assert_allclose(g["dx"], fd, rtol=0, atol=1e-7)
    for name in p:
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(p[name].shape):
            pp = {k: v.copy() for k, v in p.items()}
            pm = {k: v.copy() for k, v in p.items()}
            pp[name][idx] += h
            pm[name][idx] -= h
            fd[idx] = (J(x, pp) - J(x, pm)) / (2 * h)
        np.testing.assert_allclose(g["d" + name], fd, rtol=0, atol=1e-7, err_msg=name)


def test_postln_layer_matches_torch_autograd():
    x, p, B, H = _layer_case(B=2, S=5, H=4, dh=4, F_=64)
    D = x.shape[1]
    dy = _rand(*x.shape)
    tx = torch.tensor(x, requires_grad=True)
    tp = {k: torch.tensor(v, requires_grad=True) for k, v in p.items()}
    z1 = tx + _torch_attn(tx, tp["wqkv"], tp["bqkv"], tp["wout"], tp["bout"], B, H)
    h = F.layer_norm(z1, (D,), tp["ln1_g"], tp["ln1_b"], eps=1e-5)
    z2 = h + F.gelu(h @ tp["w1"] + tp["b1"], approximate="tanh") @ tp["w2"] + tp["b2"]
    y = F.layer_norm(z2, (D,), tp["ln2_g"], tp["ln2_b"], eps=1e-5)
    y.backward(torch.tensor(dy))
    y0, _ = layer.postln_layer_fwd(x, p, B, H)
    np.testing.assert_allclose(y0, y.detach().numpy(), atol=1e-12)
    g = layer.postln_layer_bwd(x, p, dy, B, H)
    np.testing.assert_allclose(g["dx"], tx.grad.numpy(), atol=1e-10)
    for name in p:
        np.testing.assert_allclose(g["d" + name], tp[name].grad.numpy(), atol=1e-10,
                                   err_msg=name)
