"""Pins of the RMS layer norm oracle (oracle/norm.py) to things other than
itself: torch's rms_norm and autograd in float64 as textbook routines, central
finite differences of the hand-derived backward, and closed forms."""

import numpy as np
import pytest
import torch

import oracle


def _data(M, d, seed, gemma):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, d)) * rng.uniform(0.2, 3.0, size=(M, 1))
    w = rng.standard_normal(d) * (0.1 if gemma else 0.3) + (0.0 if gemma else 1.0)
    return X, w


@pytest.mark.parametrize("gemma", [False, True])
def test_forward_matches_torch_rms_norm(gemma):
    X, w = _data(16, 96, 1, gemma)
    eps = 1e-6
    Y, rstd = oracle.rmsnorm_fwd(X, w, eps, plus_one=gemma)
    g = torch.tensor(1.0 + w if gemma else w)
    ref = torch.nn.functional.rms_norm(torch.tensor(X), (96,), weight=g, eps=eps).numpy()
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(rstd, 1.0 / np.sqrt((X ** 2).mean(1) + eps), rtol=1e-15)


@pytest.mark.parametrize("gemma", [False, True])
def test_backward_matches_torch_autograd(gemma):
    X, w = _data(8, 64, 2, gemma)
    dY = np.random.default_rng(3).standard_normal(X.shape)
    eps = 1e-5
    x = torch.tensor(X, requires_grad=True)
    g = torch.tensor(1.0 + w if gemma else w)
    torch.nn.functional.rms_norm(x, (64,), weight=g, eps=eps).backward(torch.tensor(dY))
    dX = oracle.rmsnorm_bwd(X, w, eps, dY, plus_one=gemma)
    assert np.allclose(dX, x.grad.numpy(), rtol=1e-12, atol=1e-13)


def test_backward_by_finite_differences():
    X, w = _data(3, 24, 4, False)
    dY = np.random.default_rng(5).standard_normal(X.shape)
    eps, h = 1e-5, 1e-6
    dX = oracle.rmsnorm_bwd(X, w, eps, dY)
    fd = np.zeros_like(X)
    for i in range(X.shape[0]):
        for j in range(X.shape[1]):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, j] += h
            Xm[i, j] -= h
            fd[i, j] = (np.sum(oracle.rmsnorm_fwd(Xp, w, eps)[0] * dY) - np.sum(oracle.rmsnorm_fwd(Xm, w, eps)[0] * dY)) / (2 * h)
    assert np.allclose(dX, fd, rtol=1e-6, atol=1e-8)


def test_closed_forms():
    # a constant row c normalises to sign(c) * g / sqrt(1 + eps / c^2); the Gemma gain with w = 0 is 1
    c, d, eps = -2.5, 32, 1e-6
    X = np.full((1, d), c)
    Y, rstd = oracle.rmsnorm_fwd(X, np.zeros(d), eps, plus_one=True)
    assert np.allclose(Y, -1.0 / np.sqrt(1.0 + eps / c ** 2), rtol=1e-15)
    # scale invariance up to eps, and the gradient is orthogonal to x (the output ignores the row's scale)
    X, w = _data(4, 48, 6, False)
    Y1, _ = oracle.rmsnorm_fwd(X, w, 0.0)
    Y2, _ = oracle.rmsnorm_fwd(7.0 * X, w, 0.0)
    assert np.allclose(Y1, Y2, rtol=1e-13)
    dX = oracle.rmsnorm_bwd(X, w, 0.0, np.random.default_rng(7).standard_normal(X.shape))
    assert np.allclose(np.sum(dX * X, axis=1), 0.0, atol=1e-12)
