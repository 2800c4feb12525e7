"""The seeded workload generator: determinism, shapes, distributions, FLOP counts."""
import torch

from synth import WORKLOADS, Workload, make_inputs, workload


def test_flop_counts_of_the_five_workloads():
    want = {
        "mlp_fwd_T128_D256_F1024_t2": 134_217_728,
        "attn_fwd_B4_S1024_D1024_H16_t4": 42_958_061_568,
        "mlp_fwdbwd_T8192_D3072_F12288_t8": 3_710_851_743_744,
        "mlp_fwdbwd_T8192_D7168_F28672_t8": 20_203_526_160_384,
        "layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8": 10_308_122_836_992,
    }
    assert {k: w.flops() for k, w in WORKLOADS.items()} == want


def test_inputs_are_seeded_bf16_with_the_stated_distributions():
    w = Workload("t", "layer_fwdbwd", batch=2, seq=64, hidden=256, ffn=1024, heads=4,
                 head_dim=64, t=2)
    a = make_inputs(w, seed=0)
    b = make_inputs(w, seed=0)
    c = make_inputs(w, seed=1)
    for k in a:
        assert a[k].dtype == torch.bfloat16
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["x"], c["x"])
    assert a["x"].shape == (128, 256) and a["wqkv"].shape == (256, 768)
    assert a["w1"].shape == (256, 1024) and a["w2"].shape == (1024, 256)
    assert abs(a["x"].float().std().item() - 1.0) < 0.02
    assert abs(a["w1"].float().std().item() - 0.02) < 0.001
    assert torch.count_nonzero(a["b1"]) == 0 and torch.all(a["ln1_g"] == 1)
    r = make_inputs(w, seed=0, random_affine=True)
    assert torch.equal(r["x"], a["x"]) and torch.count_nonzero(r["b1"]) > 0


def test_mlp_fwd_workload_has_no_dy():
    a = make_inputs(workload("mlp_fwd_T128_D256_F1024_t2"))
    assert "dy" not in a and a["x"].shape == (128, 256)
