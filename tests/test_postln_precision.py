"""Why the post-LN backward carries its gradient chain in fp32 (CPU only).

In the post-LN layer the gradient crosses LN2, the MLP, LN1 and attention in
a chain dz2 -> dh -> dz1, with a residual addition after each sublayer.  This
test follows that chain in fp64 with the oracle's functions and rounds where
a kernel would store: to bf16 at every link, or only the GEMM operands to
bf16 with the links themselves kept in fp32 (the library's scheme).  Against
the exact result, the first exceeds the per-element parity bound on dx for
this case and the second stays well inside it.
"""
import numpy as np
import torch

from oracle import attention, core, layer, mlp
from synth import Workload, make_inputs, to_f64

PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")


def _bf16(a):
    return torch.from_numpy(a).to(torch.bfloat16).double().numpy()


def _same(a):
    return a


def test_bf16_chain_breaks_the_bound_fp32_chain_meets_it():
    w = Workload("postln", "layer_fwdbwd", batch=2, seq=96, hidden=512, ffn=2048, heads=8,
                 head_dim=64, t=8)
    inp = make_inputs(w, seed=17, random_affine=True)
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x, dy = to_f64(inp["x"]), to_f64(inp["dy"])
    exact = layer.postln_layer_bwd(x, p, dy, w.batch, w.heads)["dx"]
    _, sv = layer.postln_layer_fwd(x, p, w.batch, w.heads)

    def chain(store_link, store_operand):
        dz2, _, _ = core.layernorm_bwd(dy, sv["z2"], p["ln2_g"], sv["mean2"], sv["rstd2"])
        gm = mlp.mlp_bwd(sv["h"], p["w1"], p["b1"], p["w2"], store_operand(dz2))
        dh = store_link(store_link(dz2) + gm["dx"])
        dz1, _, _ = core.layernorm_bwd(dh, sv["z1"], p["ln1_g"], sv["mean1"], sv["rstd1"])
        ga = attention.attn_bwd(x, p["wqkv"], p["bqkv"], p["wout"], store_operand(dz1), w.batch,
                                w.heads)
        return _bf16(store_link(dz1) + ga["dx"])      # dx itself is stored in bf16

    bound = 1e-2 * np.abs(exact).max() + 1e-3            # the per-element parity bound
    err_bf16_links = np.abs(chain(_bf16, _bf16) - exact).max()
    err_fp32_links = np.abs(chain(_same, _bf16) - exact).max()
    assert err_bf16_links > bound
    assert err_fp32_links < 0.5 * bound
