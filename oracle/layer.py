"""Unsharded transformer layer, forward and backward (fp64 NumPy).

Test infrastructure only (see the package docstring).

Pre-LN placement ("The layernorm placement the paper flags as critical":
LayerNorm before each sublayer, applied to the residual stream):
    h = x + Attn(LN1(x));   y = h + MLP(LN2(h)).
Post-LN placement (the original transformer's, the other arm of the same
passage: LayerNorm after the residual addition):
    h = LN1(x + Attn(x));   y = LN2(h + MLP(h)).
No final LayerNorm, no embedding, dropout off.
"""
from __future__ import annotations

from .attention import attn_bwd, attn_fwd
from .core import layernorm_bwd, layernorm_fwd
from .mlp import mlp_bwd, mlp_fwd


def layer_fwd(x, p, batch: int, heads: int, causal: bool = True, eps: float = 1e-5):
    """p holds ln1_g, ln1_b, wqkv, bqkv, wout, bout, ln2_g, ln2_b, w1, b1, w2, b2.

    Returns (y, saved) with the intermediates the library also saves.
    """
    u1, mean1, rstd1 = layernorm_fwd(x, p["ln1_g"], p["ln1_b"], eps)
    h, sa = attn_fwd(u1, p["wqkv"], p["bqkv"], p["wout"], p["bout"], batch, heads, causal,
                     resid=x)
    u2, mean2, rstd2 = layernorm_fwd(h, p["ln2_g"], p["ln2_b"], eps)
    y, a, hact = mlp_fwd(u2, p["w1"], p["b1"], p["w2"], p["b2"], resid=h)
    saved = dict(u1=u1, mean1=mean1, rstd1=rstd1, qkv=sa["qkv"], o=sa["o"], lse=sa["lse"],
                 h=h, u2=u2, mean2=mean2, rstd2=rstd2, a=a, hact=hact)
    return y, saved


def layer_bwd(x, p, dy, batch: int, heads: int, causal: bool = True, eps: float = 1e-5):
    """Vector-Jacobian product of ``layer_fwd`` for upstream gradient dy.

    y = h + MLP(LN2(h)) gives dh = dy + LN2^T(MLP^T(dy));
    h = x + Attn(LN1(x)) gives dx = dh + LN1^T(Attn^T(dh)).
    Returns a dict with dx and the gradient of every parameter.
    """
    u1, mean1, rstd1 = layernorm_fwd(x, p["ln1_g"], p["ln1_b"], eps)
    h, _ = attn_fwd(u1, p["wqkv"], p["bqkv"], p["wout"], p["bout"], batch, heads, causal,
                    resid=x)
    u2, mean2, rstd2 = layernorm_fwd(h, p["ln2_g"], p["ln2_b"], eps)

    gm = mlp_bwd(u2, p["w1"], p["b1"], p["w2"], dy)
    du2_x, dln2_g, dln2_b = layernorm_bwd(gm["dx"], h, p["ln2_g"], mean2, rstd2)
    dh = dy + du2_x

    ga = attn_bwd(u1, p["wqkv"], p["bqkv"], p["wout"], dh, batch, heads, causal)
    du1_x, dln1_g, dln1_b = layernorm_bwd(ga["dx"], x, p["ln1_g"], mean1, rstd1)
    dx = dh + du1_x
    return {
        "dx": dx, "dh": dh,
        "dln1_g": dln1_g, "dln1_b": dln1_b,
        "dwqkv": ga["dwqkv"], "dbqkv": ga["dbqkv"],
        "dwout": ga["dwout"], "dbout": ga["dbout"],
        "dln2_g": dln2_g, "dln2_b": dln2_b,
        "dw1": gm["dw1"], "db1": gm["db1"], "dw2": gm["dw2"], "db2": gm["db2"],
    }


# ---------------------------------------------------------------------------------------
# Post-LN variant (the original transformer placement the pages contrast with pre-LN in
# "The layernorm placement the paper flags as critical": LayerNorm after the residual
# addition):  z1 = x + Attn(x);  h = LN1(z1);  z2 = h + MLP(h);  y = LN2(z2).

def postln_layer_fwd(x, p, batch: int, heads: int, causal: bool = True, eps: float = 1e-5):
    """Returns (y, saved) for the post-LN layer."""
    z1, sa = attn_fwd(x, p["wqkv"], p["bqkv"], p["wout"], p["bout"], batch, heads, causal,
                      resid=x)
    h, mean1, rstd1 = layernorm_fwd(z1, p["ln1_g"], p["ln1_b"], eps)
    z2, a, hact = mlp_fwd(h, p["w1"], p["b1"], p["w2"], p["b2"], resid=h)
    y, mean2, rstd2 = layernorm_fwd(z2, p["ln2_g"], p["ln2_b"], eps)
    saved = dict(z1=z1, mean1=mean1, rstd1=rstd1, qkv=sa["qkv"], o=sa["o"], lse=sa["lse"],
                 h=h, z2=z2, mean2=mean2, rstd2=rstd2, a=a, hact=hact)
    return y, saved


def postln_layer_bwd(x, p, dy, batch: int, heads: int, causal: bool = True, eps: float = 1e-5):
    """Vector-Jacobian product of ``postln_layer_fwd``.

    dz2 = LN2^T(dy);  dh = dz2 + MLP^T(dz2);  dz1 = LN1^T(dh);  dx = dz1 + Attn^T(dz1).
    """
    z1, _ = attn_fwd(x, p["wqkv"], p["bqkv"], p["wout"], p["bout"], batch, heads, causal,
                     resid=x)
    h, mean1, rstd1 = layernorm_fwd(z1, p["ln1_g"], p["ln1_b"], eps)
    z2, _, _ = mlp_fwd(h, p["w1"], p["b1"], p["w2"], p["b2"], resid=h)
    _, mean2, rstd2 = layernorm_fwd(z2, p["ln2_g"], p["ln2_b"], eps)

    dz2, dln2_g, dln2_b = layernorm_bwd(dy, z2, p["ln2_g"], mean2, rstd2)
    gm = mlp_bwd(h, p["w1"], p["b1"], p["w2"], dz2)
    dh = dz2 + gm["dx"]
    dz1, dln1_g, dln1_b = layernorm_bwd(dh, z1, p["ln1_g"], mean1, rstd1)
    ga = attn_bwd(x, p["wqkv"], p["bqkv"], p["wout"], dz1, batch, heads, causal)
    return {
        "dx": dz1 + ga["dx"], "dh": dh,
        "dln1_g": dln1_g, "dln1_b": dln1_b,
        "dwqkv": ga["dwqkv"], "dbqkv": ga["dbqkv"],
        "dwout": ga["dwout"], "dbout": ga["dbout"],
        "dln2_g": dln2_g, "dln2_b": dln2_b,
        "dw1": gm["dw1"], "db1": gm["db1"], "dw2": gm["dw2"], "db2": gm["db2"],
    }
