"""CPU fp64 oracle of the tensor-parallel transformer sublayer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
bench's CPU-baseline leg may import this package.  The CUDA library never
calls it, links it or falls back to it, and it shares no code with that
library: the two meet only through the seeded inputs of the ``synth``
module.

What it computes (Megatron-LM, Shoeybi et al. 2019, as described on the pages
"Megatron-LM: what the tensor parallelism paper actually says" and
"Megatron-LM interactive explainer"):

* ``core``     GeLU (tanh form), its derivative, LayerNorm forward/backward,
               row softmax.
* ``mlp``      the UNSHARDED feed-forward sublayer ``GeLU(x W1 + b1) W2 + b2``
               ("How transformer layers actually decompose") and its
               vector-Jacobian product.
* ``attention`` the UNSHARDED causal multi-head self-attention sublayer
               ("The attention heads split") and its vector-Jacobian product.
* ``layer``    the pre-LN layer ("The layernorm placement the paper flags as
               critical"): h = x + Attn(LN1(x)); y = h + MLP(LN2(h)).
* ``sharded``  the method itself, step by step as the pages state it:
               column-split W1 / QKV by head, local GeLU / local heads,
               row-split W2 / Wout, sum of the t partial outputs.  Used to pin
               that sharding is only a re-association of the definition.
* ``layout``   the shard-packed weight layouts the library takes.

Everything is NumPy float64 on inputs that are exact bf16 values.  Matrix
products use NumPy's BLAS as a library primitive; no blocking, fusion or
reordering beyond the written definition.

Pins (``tests/test_oracle_*.py``, all ``-m "not gpu"``): brute-force scalar
loops on tiny shapes, central finite differences for every gradient, fp64
``torch`` library routines (``gelu(approximate="tanh")``, ``layer_norm``,
``scaled_dot_product_attention``, autograd) as independent references,
closed forms (GeLU(0) = 0, GeLU'(0) = 1/2, single-key softmax, uniform
softmax, constant-row LayerNorm), the exact-erf GeLU bound, the sharding
identity for t in {1, 2, 4, 8}, the GeLU-locality identity with its row-split
negative control, and the 30B FFN weight size the pages print.
No function here is "parity unpinned".
"""
from . import core, mlp, attention, layer, sharded, layout  # noqa: F401
