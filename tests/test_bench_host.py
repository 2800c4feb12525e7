"""Host-side figures of bench.py (CPU only): the recomputation cost it
reports, and the config block both arms share."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from synth import workload  # noqa: E402

LAYER = "layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8"


def test_recompute_flops_is_the_forward_without_the_second_mlp_product():
    """The recomputing backward re-runs the forward except y = H W2 (+ b2 + h):
    forward FLOPs (a third of the counted fwd+bwd) minus 2 T D F."""
    w = workload("layer_recompute_fwdbwd_B4_S2048_D4096_H32_F16384_t8")
    fwd = w.flops() // 3
    assert bench.recompute_flops(w) == fwd - 2 * w.tokens * w.hidden * w.ffn
    # 8 T D^2 (projections) + 4 dh B H S(S+1)/2 (causal core) + 2 T D F (W1)
    T, D, F = w.tokens, w.hidden, w.ffn
    core = 4 * w.head_dim * w.batch * w.heads * w.seq * (w.seq + 1) // 2
    assert bench.recompute_flops(w) == 8 * T * D * D + core + 2 * T * D * F


def test_both_arms_report_the_same_workload_identity():
    w = workload(LAYER)
    c = bench.base_config(w, 1)
    assert c["workload"] == LAYER and c["flop_per_step"] == w.flops()
    assert (c["batch"], c["seq"], c["hidden"], c["ffn"], c["heads"], c["head_dim"], c["t"]) == \
        (4, 2048, 4096, 16384, 32, 128, 8)
    # Counted work of the layer step: MLP 12TDF = 6.597 T, projections 24TD^2 =
    # 3.299 T, causal core 3 x 4 dh B H S(S+1)/2 = 0.413 T.
    assert c["flop_per_step"] == 10_308_122_836_992
