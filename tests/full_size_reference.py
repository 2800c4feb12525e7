"""The fp64 oracle of the pre-LN layer at its full workload size, computed
once per test process and shared by the test files that compare against it
(the single-GPU layer and the one-shard-per-rank layer)."""
import functools

from oracle import layer as olayer
from synth import make_inputs, to_f64, workload

PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2",
          "b2")
LAYER = "layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8"


@functools.lru_cache(maxsize=1)
def pre_ln_layer():
    """(workload, bf16 inputs, oracle y, oracle saved activations, oracle gradients)."""
    w = workload(LAYER)
    inp = make_inputs(w)
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x = to_f64(inp["x"])
    y, saved = olayer.layer_fwd(x, p, w.batch, w.heads, w.causal, w.ln_eps)
    grads = olayer.layer_bwd(x, p, to_f64(inp["dy"]), w.batch, w.heads, w.causal, w.ln_eps)
    return w, inp, y, saved, grads
