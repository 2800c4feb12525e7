"""Standalone LayerNorm forward / backward timing against a plain device copy.

    python bench_layernorm.py [T] [D] [reps]

Times tp_layernorm_fwd and tp_layernorm_bwd (with and without the residual
gradient) through the Python binding on seeded random bf16 inputs of T rows x D,
each launch after a 256 MB L2 flush, with CUDA events on the launch stream
(median of `reps`), and torch's copy of one T x D bf16 tensor on the same device
as the bandwidth reference.  Bytes are the algorithmic ones: the forward reads x
and writes y; the backward reads dy, x (and dres) and writes dx.
"""
import statistics
import sys

import torch

import tensor_transformer_layer_column_b200 as tl


def main():
    T = int(sys.argv[1]) if len(sys.argv) > 1 else 32768
    D = int(sys.argv[2]) if len(sys.argv) > 2 else 4096
    reps = int(sys.argv[3]) if len(sys.argv) > 3 else 20
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device="cpu").manual_seed(5)
    bf = torch.bfloat16
    x = torch.randn(T, D, generator=gen).to(bf).to(dev)
    dy = torch.randn(T, D, generator=gen).to(bf).to(dev)
    dres = torch.randn(T, D, generator=gen).to(bf).to(dev)
    g = (1 + 0.1 * torch.randn(D, generator=gen)).to(bf).to(dev)
    b = (0.1 * torch.randn(D, generator=gen)).to(bf).to(dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    mean = torch.empty(T, device=dev)
    rstd = torch.empty(T, device=dev)
    dg = torch.empty(D, dtype=bf, device=dev)
    db = torch.empty_like(dg)
    ws = torch.empty(tl.layernorm_bwd_workspace_size(T, D), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        out = []
        for _ in range(reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1))
        return statistics.median(out) * 1e-3   # seconds

    fwd = lambda: tl.layernorm_fwd(x, g, b, T, D, 1e-5, y, mean, rstd)
    bwd_res = lambda: tl.layernorm_bwd(dy, x, g, mean, rstd, dres, T, D, dx, dg, db, ws)
    bwd = lambda: tl.layernorm_bwd(dy, x, g, mean, rstd, None, T, D, dx, dg, db, ws)
    copy = lambda: dx.copy_(x)
    for _ in range(3):
        fwd(); bwd_res(); bwd(); copy()
    torch.cuda.synchronize()
    E = T * D * 2
    for name, fn, nbytes in (("ln_fwd", fwd, 2 * E), ("ln_bwd with dres", bwd_res, 4 * E),
                             ("ln_bwd", bwd, 3 * E), ("torch copy", copy, 2 * E)):
        t = timed(fn)
        print(f"T={T} D={D} {name}: {t * 1e6:.1f} us, {nbytes / t / 1e9:.0f} GB/s")


if __name__ == "__main__":
    main()
