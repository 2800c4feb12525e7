"""Seeded synthetic workloads for the tensor-parallel transformer sublayer.

This module is shared by the tests, the bench and the smoke check.  It holds
the five named workload shapes and a seeded generator of their inputs, and
nothing of the method's arithmetic: no GeLU, no attention, no normalisation,
no sharding.  Both the CPU oracle and the CUDA path receive the very same
bf16 values from here.

Recipe (Megatron-LM pages, "How transformer layers actually decompose" and
"The attention heads split"; the workload list fixes the distributions):

* one CPU ``torch.Generator`` seeded with ``seed`` (0 by default);
* tensors drawn in a fixed order -- x, the weights in layer order, then the
  upstream gradient dY -- each as fp32 N(0, 1) times its standard deviation,
  then rounded to nearest-even bf16;
* x ~ N(0, 1), weight matrices ~ N(0, 0.02), dY ~ N(0, 1);
* biases zero, LayerNorm gamma = 1 and beta = 0, unless ``random_affine`` is
  set, in which case a second generator (seed + 1) draws biases ~ N(0, 0.1),
  gamma ~ 1 + N(0, 0.1), beta ~ N(0, 0.1) and a residual input ~ N(0, 1), so
  that tests can pin where biases and residuals enter.

Weights are produced unsharded, in the orientation the pages use for
``output = GeLU(x W1) W2`` (weights are [in, out]): W1 [D, F], W2 [F, D],
Wqkv [D, 3D] = [Wq | Wk | Wv] with head h in columns h*dh .. (h+1)*dh-1 of each
part, Wout [D, D].  Activations are [T, D] with T = batch * seq, batch outer.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "EXTRA_WORKLOADS", "workload", "make_inputs", "to_f64"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "mlp_fwd", "attn_fwd", "mlp_fwdbwd", "layer_fwdbwd", or a test kind
    batch: int
    seq: int
    hidden: int
    ffn: int = 0
    heads: int = 0
    head_dim: int = 0
    t: int = 1
    causal: bool = True
    ln_eps: float = 1e-5

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def has_mlp(self) -> bool:
        return self.kind.startswith("mlp") or self.kind.startswith("layer")

    @property
    def has_attn(self) -> bool:
        return self.kind.startswith("attn") or self.kind.startswith("layer")

    @property
    def backward(self) -> bool:
        return self.kind.endswith("fwdbwd")

    def flops(self) -> int:
        """Algorithmic FLOPs of the workload: GEMM-like work only.

        MLP 4*T*D*F forward, attention projections 8*T*D^2 forward, causal
        core 4*dh*B*H*S(S+1)/2 forward (masked dense work not counted);
        backward counts twice the forward and no recompute.
        """
        T, D, F = self.tokens, self.hidden, self.ffn
        fwd = 0
        if self.has_mlp:
            fwd += 4 * T * D * F
        if self.has_attn:
            fwd += 8 * T * D * D
            pairs = self.seq * (self.seq + 1) // 2 if self.causal else self.seq * self.seq
            fwd += 4 * self.head_dim * self.batch * self.heads * pairs
        return 3 * fwd if self.backward else fwd


# The five workloads of the tensor-parallel sublayer, with the sizes the
# pages give (8.3B GPT-2-style width, the 30B FFN shape [7168, 28672]).
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("mlp_fwd_T128_D256_F1024_t2", "mlp_fwd", batch=2, seq=64, hidden=256, ffn=1024, t=2),
    Workload("attn_fwd_B4_S1024_D1024_H16_t4", "attn_fwd", batch=4, seq=1024, hidden=1024,
             heads=16, head_dim=64, t=4),
    Workload("mlp_fwdbwd_T8192_D3072_F12288_t8", "mlp_fwdbwd", batch=8, seq=1024, hidden=3072,
             ffn=12288, t=8),
    Workload("mlp_fwdbwd_T8192_D7168_F28672_t8", "mlp_fwdbwd", batch=4, seq=2048, hidden=7168,
             ffn=28672, t=8),
    Workload("layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8", "layer_fwdbwd", batch=4, seq=2048,
             hidden=4096, ffn=16384, heads=32, head_dim=128, t=8),
]}

# Beyond the five: a profiling case (the layer's attention sublayer at half the
# batch; inputs exceed L2 but it holds < 1 GB), the post-LN arm of the
# layer-norm placement passage at the pre-LN layer's size, and the pre-LN layer
# with activation recomputation (nothing kept between forward and backward).
EXTRA_WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("attn_fwdbwd_B2_S2048_D4096_H32_t8", "attn_fwdbwd", batch=2, seq=2048, hidden=4096,
             heads=32, head_dim=128, t=8),
    Workload("layer_postln_fwdbwd_B4_S2048_D4096_H32_F16384_t8", "layer_postln_fwdbwd", batch=4,
             seq=2048, hidden=4096, ffn=16384, heads=32, head_dim=128, t=8),
    Workload("layer_recompute_fwdbwd_B4_S2048_D4096_H32_F16384_t8", "layer_recompute_fwdbwd",
             batch=4, seq=2048, hidden=4096, ffn=16384, heads=32, head_dim=128, t=8),
]}


def workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else EXTRA_WORKLOADS[name]


def _normal(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0, random_affine: bool = False,
                with_dy: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    """Seeded bf16 CPU tensors for workload ``w`` (unsharded layout)."""
    gen = torch.Generator().manual_seed(seed)
    T, D, F = w.tokens, w.hidden, w.ffn
    out: Dict[str, torch.Tensor] = {}
    out["x"] = _normal(gen, (T, D), 1.0)
    if w.has_attn:
        out["wqkv"] = _normal(gen, (D, 3 * D), 0.02)
        out["wout"] = _normal(gen, (D, D), 0.02)
    if w.has_mlp:
        out["w1"] = _normal(gen, (D, F), 0.02)
        out["w2"] = _normal(gen, (F, D), 0.02)
    if with_dy is None:
        with_dy = w.backward
    if with_dy:
        out["dy"] = _normal(gen, (T, D), 1.0)

    g2 = torch.Generator().manual_seed(seed + 1)

    def bias(n):
        return _normal(g2, (n,), 0.1) if random_affine else torch.zeros(n, dtype=torch.bfloat16)

    def gamma(n):
        if random_affine:
            return (1.0 + 0.1 * torch.randn(n, generator=g2)).to(torch.bfloat16)
        return torch.ones(n, dtype=torch.bfloat16)

    if w.has_attn:
        out["bqkv"] = bias(3 * D)
        out["bout"] = bias(D)
    if w.has_mlp:
        out["b1"] = bias(F)
        out["b2"] = bias(D)
    if w.kind.startswith("layer"):
        out["ln1_g"], out["ln1_b"] = gamma(D), bias(D)
        out["ln2_g"], out["ln2_b"] = gamma(D), bias(D)
    elif random_affine:
        out["resid"] = _normal(g2, (T, D), 1.0)
    return out


def to_f64(t: torch.Tensor):
    """Exact widening of a bf16 tensor to a float64 NumPy array."""
    return t.to(torch.float64).numpy()
