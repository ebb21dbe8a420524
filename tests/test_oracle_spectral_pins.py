"""Pins of the spectral-compression oracle ("Nitrobrew tweet analysis": thread item 6/8 and
the evaluation table's "SVD-Nitrobrew" row, k floats per token).

Expected values come from matrices built with a known SVD (random orthogonal factors and
chosen singular values), from closed forms, and from the uncompressed loss — not from the
oracle's own SVD call.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import spectral as sp


def known_svd(rng, V, d, s):
    """W = U diag(s) Q^T with orthonormal U [V, d], Q [d, d]."""
    U, _ = np.linalg.qr(rng.standard_normal((V, d)))
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return U @ np.diag(s) @ Q.T, U, Q


def test_top_subspace_and_eckart_young():
    rng = np.random.default_rng(0)
    V, d, k = 60, 12, 5
    s = np.array([9.0, 7.5, 6.0, 5.0, 4.2, 1.0, 0.9, 0.7, 0.5, 0.3, 0.2, 0.1])
    W, _, Q = known_svd(rng, V, d, s)
    Vk, sig = sp.spectral_basis(W, k)
    np.testing.assert_allclose(sig, s[:k], rtol=1e-12)
    # the basis spans the top-k right singular subspace that was built in
    np.testing.assert_allclose(Vk @ Vk.T, Q[:, :k] @ Q[:, :k].T, atol=1e-12)
    np.testing.assert_allclose(Vk.T @ Vk, np.eye(k), atol=1e-12)
    # truncation error: ||W - W V_k V_k^T||_F^2 = sum of the dropped sigma^2
    R = W - W @ Vk @ Vk.T
    assert (R ** 2).sum() == pytest.approx((s[k:] ** 2).sum(), rel=1e-10)


def test_closed_form_diagonal():
    # W = [[3, 0], [0, 1], [0, 0]]: V_1 = +-e1, W' = +-[3, 0, 0]^T, h' = +-h_1
    W = np.array([[3.0, 0.0], [0.0, 1.0], [0.0, 0.0]])
    h = np.array([[2.0, -5.0], [0.5, 4.0]])
    hp, Wp, Vk = sp.compress_teacher(h, W, 1)
    sgn = np.sign(Vk[0, 0])
    np.testing.assert_allclose(Vk[:, 0], sgn * np.array([1.0, 0.0]), atol=1e-15)
    np.testing.assert_allclose(Wp[:, 0], sgn * np.array([3.0, 0.0, 0.0]), atol=1e-14)
    np.testing.assert_allclose(hp[:, 0], sgn * h[:, 0], atol=1e-14)
    # logits of the compressed pair: keep only the first coordinate
    np.testing.assert_allclose(hp @ Wp.T, np.array([[6.0, 0.0, 0.0], [1.5, 0.0, 0.0]]), atol=1e-13)


def test_full_rank_and_exact_low_rank_are_lossless():
    rng = np.random.default_rng(1)
    V, d, N = 80, 10, 7
    W = rng.standard_normal((V, d))
    h = rng.standard_normal((N, d))
    hp, Wp, _ = sp.compress_teacher(h, W, d)
    np.testing.assert_allclose(hp @ Wp.T, h @ W.T, atol=1e-11)
    # rank-4 teacher kept at k = 4: still exact
    W4 = rng.standard_normal((V, 4)) @ rng.standard_normal((4, d))
    hp, Wp, _ = sp.compress_teacher(h, W4, 4)
    np.testing.assert_allclose(hp @ Wp.T, h @ W4.T, atol=1e-11)


@pytest.mark.parametrize("beta", [0.0, 1.0, 0.5])
def test_compressed_loss_equals_loss_of_projected_teacher(beta):
    """The loss on (h_t', W_t') is the loss of the rank-k teacher W_t V_k V_k^T, and equals
    the uncompressed loss at full rank."""
    rng = np.random.default_rng(2)
    N, V, d_s, d_t, k = 9, 70, 6, 8, 3
    h_s, h_t = rng.standard_normal((N, d_s)), rng.standard_normal((N, d_t))
    W_s, W_t = rng.standard_normal((V, d_s)), rng.standard_normal((V, d_t))
    labels = rng.integers(0, V, N)
    hp, Wp, Vk = sp.compress_teacher(h_t, W_t, k)
    a = oracle.forward(h_s, W_s, hp, Wp, labels, beta, 1.2)
    b = oracle.forward(h_s, W_s, h_t, W_t @ Vk @ Vk.T, labels, beta, 1.2)
    np.testing.assert_allclose(a["loss_tok"], b["loss_tok"], rtol=1e-10, atol=1e-13)
    hp, Wp, _ = sp.compress_teacher(h_t, W_t, d_t)
    c = oracle.forward(h_s, W_s, hp, Wp, labels, beta, 1.2)
    d = oracle.forward(h_s, W_s, h_t, W_t, labels, beta, 1.2)
    np.testing.assert_allclose(c["loss_tok"], d["loss_tok"], rtol=1e-9, atol=1e-12)


def test_codes_are_coordinates_in_the_basis():
    rng = np.random.default_rng(3)
    W, _, _ = known_svd(rng, 40, 6, np.array([5.0, 4.0, 3.0, 2.0, 1.0, 0.5]))
    Vk, _ = sp.spectral_basis(W, 6)
    h = rng.standard_normal((5, 6))
    # full basis: h is recovered from its code; norms are kept
    np.testing.assert_allclose(sp.project(h, Vk) @ Vk.T, h, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(sp.project(h, Vk), axis=1), np.linalg.norm(h, axis=1),
                               rtol=1e-12)
    with pytest.raises(ValueError):
        sp.spectral_basis(W, 0)
    with pytest.raises(ValueError):
        sp.spectral_basis(W, 7)
