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


def test_hbm_bytes_of_the_layer_step():
    w = workload(LAYER)
    b = bench.hbm_bytes_per_step(w)
    T, D, F = w.tokens, w.hidden, w.ffn
    assert b["ln_fwd"] == 2 * 4 * T * D + 16 * T                # 2 x (64 MiB in + 64 MiB out) + stats
    assert b["ln_bwd"] == 16 * T * D + 16 * T                   # 2 x (3 reads + 1 write of [T][D])
    # db1 / dbqkv partial rows (one per 32 rows, fp32) read, the sums written
    assert b["colsum"] == 4 * (T // 32) * (F + 3 * D) + 2 * (F + 3 * D)
    assert b["cast"] == 12 * D * D                              # Wqkv read + written, once
    assert abs(b["ln_bwd"] / 2**20 - 512.125) < 1e-9            # 512 MiB of rows + 128 KiB of stats
    assert bench.hbm_bytes_per_step(workload("mlp_fwdbwd_T8192_D3072_F12288_t8")) == {}


PEAKS = {"hbm_gbs": 6425.6, "bf16_tflops": 1713.1, "bf16_tflops_sustained": 1430.5}


def test_peak_follows_the_sampled_clock():
    """Burst figure when the SM clock held at its maximum, sustained when it sagged."""
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    sagged = {"sm_mhz": 1455.0, "sm_max_mhz": 1965.0}
    assert bench.choose_peak(PEAKS, at_max) == (1713.1, "bf16_tflops")
    assert bench.choose_peak(PEAKS, {"sm_mhz": 1890.0, "sm_max_mhz": 1965.0})[0] == 1713.1
    assert bench.choose_peak(PEAKS, sagged) == (1430.5, "bf16_tflops_sustained")
    # No clock record: the larger denominator.
    assert bench.choose_peak(PEAKS, {"sm_mhz": None, "sm_max_mhz": None})[0] == 1713.1


def test_roofline_fraction_of_a_recorded_run():
    """The first round's c5 line: 9.896 TFLOP of GEMM work per step in 7.587 ms
    at 1965 MHz is 1304 TFLOP/s, 0.76 of the burst figure (not 0.91 of the
    sustained one)."""
    gemm_flop = 12 * 8192 * 4096 * 16384 + 24 * 8192 * 4096 * 4096
    achieved = gemm_flop / 7.586649605631829e-3 / 1e12
    peak, name = bench.choose_peak(PEAKS, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert abs(achieved - 1304.3) < 0.1
    assert abs(achieved / peak - 0.761) < 1e-3 and name == "bf16_tflops"
    assert bench.clock_normalised(achieved, {"sm_mhz": 1455.0, "sm_max_mhz": 1965.0}) == \
        achieved * 1965.0 / 1455.0


def test_step_time_is_the_median_of_per_step_durations():
    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    evs = [Ev(t) for t in (0.0, 9.0, 18.5, 27.0, 45.0)]   # steps 9, 9.5, 8.5, 18
    assert bench.median_step_ms(evs) == 9.25
