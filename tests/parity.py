"""Tolerance checks of the CUDA path against the fp64 oracle.

Per element |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3 and relative L2
error <= 5e-3, on every output and gradient.
"""
import numpy as np
import torch

ATOL_FRAC = 1e-2
ATOL_ABS = 1e-3
REL_L2 = 5e-3


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to(torch.float64).cpu().numpy()


def check(name: str, gpu, ref: np.ndarray):
    g = f64(gpu).reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    err = np.abs(g - ref)
    bound = ATOL_FRAC * np.abs(ref).max() + ATOL_ABS
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= bound, f"{name}: max err {err.max():.3e} > {bound:.3e} (relL2 {rel:.3e})"
    assert rel <= REL_L2, f"{name}: relL2 {rel:.3e} > {REL_L2}"
    return float(rel)
