"""Pins for the oracle's Hessian, damping and factor: brute force on integer data (exact),
closed forms, and residual identities."""

import numpy as np
import pytest

from oracle import factor, hessian


def test_hessian_integer_brute_force():
    rng = np.random.default_rng(0)
    X = rng.integers(-3, 4, size=(7, 5)).astype(np.float16)
    H = hessian.hessian(X, chunk=3)
    n, d = X.shape
    for i in range(d):
        for j in range(d):
            acc = 0
            for t in range(n):
                acc += int(X[t, i]) * int(X[t, j])
            assert H[i, j] == 2 * acc


def test_hessian_symmetric_psd_rank_and_additive():
    rng = np.random.default_rng(1)
    X = (rng.standard_normal((12, 20))).astype(np.float16)
    H = hessian.hessian(X)
    assert np.array_equal(H, H.T)
    ev = np.linalg.eigvalsh(H)
    assert ev.min() > -1e-9 * ev.max()
    assert np.sum(ev > 1e-9 * ev.max()) <= 12          # rank <= n_tokens
    Xi = rng.integers(-5, 6, size=(30, 6)).astype(np.float16)
    assert np.array_equal(hessian.hessian(Xi), hessian.hessian(Xi[:13]) + hessian.hessian(Xi[13:]))
    rows, cols = np.array([0, 3, 5]), np.array([1, 2])
    assert np.array_equal(hessian.hessian_entries(Xi, rows, cols), hessian.hessian(Xi)[np.ix_(rows, cols)])


def test_damping_closed_form_and_failure():
    H = np.diag([1.0, 2.0, 3.0, 6.0])
    Hd, lam = factor.damp(H, 0.01)
    assert lam == pytest.approx(0.01 * 3.0, rel=0, abs=1e-15)
    assert np.array_equal(Hd, H + lam * np.eye(4))
    with pytest.raises(factor.NotPositiveDefinite):
        factor.damp(np.zeros((4, 4)), 0.01)
    with pytest.raises(factor.NotPositiveDefinite):
        factor.damp(H, 0.0)


def test_damping_makes_rank_deficient_hessian_pd():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((5, 16)).astype(np.float16)
    H = hessian.hessian(X)
    with pytest.raises(np.linalg.LinAlgError):
        np.linalg.cholesky(H)
    Hd, _ = factor.damp(H, 0.01)
    L = np.linalg.cholesky(Hd)
    assert np.all(np.diag(L) > 0)


def test_upper_factor_2x2_closed_form():
    a, b, c = 4.0, 1.5, 3.0
    U = factor.upper_chol_of_inverse(np.array([[a, b], [b, c]]))
    det = a * c - b * b
    u11 = np.sqrt(c / det)
    u12 = -b / (det * u11)
    u22 = 1.0 / np.sqrt(c)
    assert np.allclose(U, [[u11, u12], [0.0, u22]], rtol=1e-14, atol=0)


def test_upper_factor_diagonal():
    h = np.array([2.0, 5.0, 0.5])
    U = factor.upper_chol_of_inverse(np.diag(h))
    assert np.allclose(U, np.diag(1 / np.sqrt(h)), rtol=1e-15, atol=0)


@pytest.mark.parametrize("d,n", [(8, 100), (64, 40), (200, 1000)])
def test_upper_factor_residual_and_routes_agree(d, n):
    rng = np.random.default_rng(d)
    X = (rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))).astype(np.float16)
    Hd, _ = factor.damp(hessian.hessian(X), 0.01)
    U = factor.upper_chol_of_inverse(Hd)
    assert np.array_equal(U, np.triu(U)) and np.all(np.diag(U) > 0)
    R = U.T @ U @ Hd - np.eye(d)
    assert np.max(np.abs(R)) <= 1e-9
    U2 = factor.upper_chol_of_inverse_reversed(Hd)
    assert np.max(np.abs(U - U2)) <= 1e-10 * np.max(np.abs(U))


@pytest.mark.parametrize("act_order", [False, True])
def test_prepare_u_is_the_upper_factor_of_the_damped_ordered_inverse(act_order):
    """The (perm, U) pair the GPU's inverse factor is compared with: perm is the processing
    order (identity, or diag(H) descending with ties by lower index), and U is the unique upper
    triangular factor with a positive diagonal of (P H P + lambda I)^-1, lambda = 0.01 mean(diag H)."""
    from oracle import gptq as og
    rng = np.random.default_rng(11)
    X = rng.standard_normal((300, 24)) * np.exp(rng.standard_normal(24))
    X[:, 5] = X[:, 9]                      # a tie on the diagonal and a rank-deficient pair
    H = 2.0 * X.T @ X
    perm, U = og.prepare_u(H, 0.01, act_order)
    d = H.shape[0]
    diag = np.diag(H)
    if act_order:
        assert sorted(perm.tolist()) == list(range(d))
        dp = diag[perm]
        assert np.all(np.diff(dp) <= 0)
        for a in range(d - 1):             # equal keys keep index order
            if dp[a] == dp[a + 1]:
                assert perm[a] < perm[a + 1]
        assert list(perm).index(5) < list(perm).index(9)
    else:
        assert np.array_equal(perm, np.arange(d))
    assert np.array_equal(U, np.triu(U)) and np.all(np.diag(U) > 0)
    Hd = H[np.ix_(perm, perm)] + 0.01 * np.mean(diag) * np.eye(d)
    assert np.max(np.abs(U.T @ U @ Hd - np.eye(d))) <= 1e-9
