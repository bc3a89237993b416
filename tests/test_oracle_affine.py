"""Pins of the oracle's closed-form centred affine fit.

Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
section "A closed-form fit avoids retraining from scratch": teacher outputs and
converted linear outputs are accumulated across scenes, tokens, heads and
views, and a centred affine correction is fitted by regularised least squares
in float64. The page prints no numbers, so each pin is a closed form, a
library routine or an invariant.
"""
import numpy as np
import pytest

import oracle


def _data(seed, n=400, H=2, d=64, noise=0.0):
    r = np.random.default_rng(seed)
    X = r.standard_normal((n, H, d)) + r.standard_normal(d)   # nonzero mean: the centring matters
    A0 = 0.2 * r.standard_normal((H, d, d))
    b0 = r.standard_normal((H, d))
    Y = np.einsum("nhj,hij->nhi", X, A0) + b0 + noise * r.standard_normal((n, H, d))
    return X, Y, A0, b0


def test_noise_free_recovery_per_head():
    # y = A0 x + b0 exactly -> the unregularised fit returns A0, b0
    X, Y, A0, b0 = _data(1)
    A, b = oracle.affine_fit(X, Y, 0.0, per_head=True)
    np.testing.assert_allclose(A, A0, atol=1e-10)
    np.testing.assert_allclose(b, b0, atol=1e-10)


def test_pooled_equals_lstsq_on_augmented_system():
    # lam = 0: the centred fit is ordinary least squares with an intercept
    # (numpy lstsq on [x, 1] -> [y]); heads pooled as extra rows
    X, Y, _, _ = _data(2, noise=0.3)
    A, b = oracle.affine_fit(X, Y, 0.0, per_head=False)
    n, H, d = X.shape
    Xa = np.concatenate([X.reshape(n * H, d), np.ones((n * H, 1))], axis=1)
    W, *_ = np.linalg.lstsq(Xa, Y.reshape(n * H, d), rcond=None)
    np.testing.assert_allclose(A[0], W[:d].T, atol=1e-9)
    np.testing.assert_allclose(b[0], W[d], atol=1e-9)


@pytest.mark.parametrize("lam", [0.05, 1.0])
def test_ridge_normal_equations_two_pass(lam):
    # the fit from raw moments satisfies (C_xx + lam I) A^T = C_xy with the
    # covariances computed the direct way (subtract the means, then multiply)
    X, Y, _, _ = _data(3, noise=0.5)
    A, b = oracle.affine_fit(X, Y, lam, per_head=True)
    for h in range(X.shape[1]):
        xc = X[:, h] - X[:, h].mean(0)
        yc = Y[:, h] - Y[:, h].mean(0)
        cxx = xc.T @ xc / len(xc)
        cxy = xc.T @ yc / len(xc)
        np.testing.assert_allclose((cxx + lam * np.eye(64)) @ A[h].T, cxy, atol=1e-10)
        np.testing.assert_allclose(b[h], Y[:, h].mean(0) - A[h] @ X[:, h].mean(0), atol=1e-10)


def test_large_regularisation_limit():
    # lam -> inf: A -> C_xy / lam -> 0 and b -> mean(y)
    X, Y, _, _ = _data(4, noise=0.1)
    A, b = oracle.affine_fit(X, Y, 1e9, per_head=False)
    assert np.abs(A).max() < 1e-7
    np.testing.assert_allclose(b[0], Y.reshape(-1, 64).mean(0), atol=1e-6)


def test_accumulation_across_calls():
    # moments of two scenes added == moments of both scenes at once
    X, Y, _, _ = _data(5, n=300, noise=0.2)
    m = oracle.affine_moments_add(oracle.affine_moments(X[:120], Y[:120]), oracle.affine_moments(X[120:], Y[120:]))
    A1, b1 = oracle.affine_solve(m, 0.1)
    A2, b2 = oracle.affine_fit(X, Y, 0.1)
    np.testing.assert_allclose(A1, A2, atol=1e-12)
    np.testing.assert_allclose(b1, b2, atol=1e-12)


def test_pooled_equals_per_head_when_heads_agree():
    r = np.random.default_rng(6)
    x1 = r.standard_normal((200, 1, 64))
    y1 = 0.5 * x1[..., ::-1] + 1.0 + 0.1 * r.standard_normal((200, 1, 64))
    X = np.repeat(x1, 3, axis=1)
    Y = np.repeat(y1, 3, axis=1)
    Ap, bp = oracle.affine_fit(X, Y, 0.01, per_head=False)
    Ah, bh = oracle.affine_fit(X, Y, 0.01, per_head=True)
    for h in range(3):
        np.testing.assert_allclose(Ah[h], Ap[0], atol=1e-10)
        np.testing.assert_allclose(bh[h], bp[0], atol=1e-10)


def test_fit_reduces_error_of_linear_stage_against_dense():
    # on a tiny geometry: with lam = 0 the identity map is one of the candidate
    # affine maps, so the least-squares correction of the linear stage towards
    # dense attention (the teacher) cannot have a larger mean squared error
    g = oracle.Geom(4, 16, 16, 2)
    r = np.random.default_rng(7)
    q, k, v = (r.standard_normal((g.n_tokens, 2, 64)) for _ in range(3))
    eye = np.repeat(np.eye(64)[None], 2, axis=0)
    zero = np.zeros((2, 64))
    x = oracle.linear_stage(q, k, v, g, eye, zero)
    y = np.stack([oracle.dense_attention(q[:, h], k[:, h], v[:, h]) for h in range(2)], axis=1)
    A, b = oracle.affine_fit(x, y, 0.0, per_head=True)
    corrected = np.einsum("nhj,hij->nhi", x, A) + b
    assert np.mean((corrected - y) ** 2) < np.mean((x - y) ** 2)


def test_residual_from_moments_equals_direct_error():
    # the conversion error computed from raw moments equals the mean squared
    # error of the corrected samples
    X, Y, _, _ = _data(8, noise=0.4)
    m = oracle.affine_moments(X, Y, per_head=True)
    A, b = oracle.affine_solve(m, 0.05)
    err = oracle.affine_residual(m, A, b)
    for h in range(X.shape[1]):
        direct = np.mean(np.sum((X[:, h] @ A[h].T + b[h] - Y[:, h]) ** 2, axis=1))
        assert abs(err[h] - direct) < 1e-9 * max(1.0, direct)
    # an exact fit leaves no error
    X0, Y0, _, _ = _data(9)
    m0 = oracle.affine_moments(X0, Y0, per_head=True)
    A0, b0 = oracle.affine_solve(m0, 0.0)
    assert (np.abs(oracle.affine_residual(m0, A0, b0)) < 1e-8).all()


def test_allocation_takes_the_lowest_errors():
    errors = [0.5, 0.1, 0.3, 0.1, 0.9, 0.2]
    # round(0.5 * 6) = 3 stages: the two 0.1 (lower index first) and 0.2
    assert oracle.allocate_layers(errors, 0.5).tolist() == [False, True, False, True, False, True]
    assert not oracle.allocate_layers(errors, 0.0).any()
    assert oracle.allocate_layers(errors, 1.0).all()
    # 0.7 x 24 = 16.8 -> 17 linear stages; with increasing errors they are the first 17
    lin = oracle.allocate_layers(np.arange(24.0), 0.7)
    assert lin.sum() == 17 and lin[:17].all()
    # ties: the lower stage index wins the last place
    assert oracle.allocate_layers([1.0, 1.0, 1.0], 1 / 3).tolist() == [True, False, False]
