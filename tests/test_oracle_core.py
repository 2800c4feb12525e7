"""Pins of the oracle's elementwise and row-wise pieces (CPU only)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import core


def test_gelu_closed_forms():
    # GeLU(0) = 0, GeLU'(0) = 1/2, GeLU(a) -> a for large a, -> 0 for very negative a.
    assert core.gelu(np.array(0.0)) == 0.0
    assert core.gelu_grad(np.array(0.0)) == 0.5
    assert abs(core.gelu(np.array(10.0)) - 10.0) < 1e-12
    assert abs(core.gelu(np.array(-10.0))) < 1e-12
    assert abs(core.gelu_grad(np.array(10.0)) - 1.0) < 1e-12


def test_gelu_within_published_bound_of_exact_gelu():
    # The tanh form approximates a * Phi(a); its largest gap is below 5e-4,
    # so a wrong constant or a dropped cubic term fails here.
    a = np.linspace(-8, 8, 40001)
    exact = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in a])
    gap = np.abs(core.gelu(a) - exact).max()
    assert 1e-4 < gap < 6e-4


def test_gelu_matches_torch_tanh_gelu_and_autograd():
    a = np.linspace(-7, 7, 1001)
    ta = torch.tensor(a, dtype=torch.float64, requires_grad=True)
    ref = F.gelu(ta, approximate="tanh")
    ref.sum().backward()
    np.testing.assert_allclose(core.gelu(a), ref.detach().numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(core.gelu_grad(a), ta.grad.numpy(), rtol=0, atol=1e-13)


def test_gelu_grad_finite_difference():
    a = np.linspace(-5, 5, 201)
    h = 1e-6
    fd = (core.gelu(a + h) - core.gelu(a - h)) / (2 * h)
    np.testing.assert_allclose(core.gelu_grad(a), fd, rtol=0, atol=1e-8)


def test_layernorm_constant_row_gives_beta():
    x = np.full((3, 16), 2.5)
    g = np.linspace(0.5, 1.5, 16)
    b = np.linspace(-1, 1, 16)
    y, mean, rstd = core.layernorm_fwd(x, g, b, 1e-5)
    np.testing.assert_array_equal(y, np.broadcast_to(b, y.shape))
    np.testing.assert_array_equal(mean, 2.5)
    np.testing.assert_allclose(rstd, 1 / math.sqrt(1e-5))


def test_layernorm_matches_torch_layer_norm_and_autograd():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(5, 24)) * 3 + 1
    g = rng.normal(size=24)
    b = rng.normal(size=24)
    dy = rng.normal(size=(5, 24))
    tx = torch.tensor(x, requires_grad=True)
    tg = torch.tensor(g, requires_grad=True)
    tb = torch.tensor(b, requires_grad=True)
    ref = F.layer_norm(tx, (24,), tg, tb, eps=1e-5)
    ref.backward(torch.tensor(dy))
    y, mean, rstd = core.layernorm_fwd(x, g, b, 1e-5)
    np.testing.assert_allclose(y, ref.detach().numpy(), rtol=0, atol=1e-12)
    dx, dg, db = core.layernorm_bwd(dy, x, g, mean, rstd)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=0, atol=1e-12)


def test_layernorm_bwd_finite_difference():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 8))
    g = rng.normal(size=8)
    b = rng.normal(size=8)
    dy = rng.normal(size=(3, 8))
    y, mean, rstd = core.layernorm_fwd(x, g, b)
    dx, dg, db = core.layernorm_bwd(dy, x, g, mean, rstd)

    def J(xx, gg, bb):
        return (core.layernorm_fwd(xx, gg, bb)[0] * dy).sum()

    h = 1e-6
    for arr, grad, args in ((x, dx, 0), (g, dg, 1), (b, db, 2)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = [x.copy(), g.copy(), b.copy()], [x.copy(), g.copy(), b.copy()]
            p[args][idx] += h
            m[args][idx] -= h
            fd[idx] = (J(*p) - J(*m)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=0, atol=1e-7)


def test_softmax_rows_single_entry_and_uniform():
    s = np.array([[3.0, -np.inf, -np.inf], [1.0, 1.0, -np.inf], [0.0, 0.0, 0.0]])
    p = core.softmax_rows(s)
    np.testing.assert_array_equal(p[0], [1.0, 0.0, 0.0])
    np.testing.assert_allclose(p[1], [0.5, 0.5, 0.0])
    np.testing.assert_allclose(p[2], [1 / 3] * 3)


@pytest.mark.parametrize("shift", [0.0, 700.0])
def test_softmax_rows_is_shift_invariant(shift):
    rng = np.random.default_rng(3)
    s = rng.normal(size=(4, 9))
    np.testing.assert_allclose(core.softmax_rows(s + shift), core.softmax_rows(s), atol=1e-15)
