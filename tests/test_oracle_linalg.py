"""Pins for the oracle's CholQR and one-sided Jacobi SVD."""

import numpy as np

from oracle import linalg


def test_cholqr_random_tall():
    rng = np.random.default_rng(0)
    for m, n in ((40, 8), (300, 72), (82, 72)):
        Y = rng.standard_normal((m, n))
        Q, R, dropped = linalg.cholqr(Y)
        assert not dropped.any()
        assert np.allclose(Q.T @ Q, np.eye(n), atol=1e-10)
        assert np.allclose(Q @ R, Y, atol=1e-10)
        assert np.allclose(np.tril(R, -1), 0)
        assert np.all(np.diag(R) > 0)


def test_cholqr_matches_householder_qr_up_to_signs():
    rng = np.random.default_rng(1)
    Y = rng.standard_normal((50, 10))
    Q, R, _ = linalg.cholqr(Y)
    Qh, Rh = np.linalg.qr(Y)
    sgn = np.sign(np.diag(Rh))
    assert np.allclose(R, Rh * sgn[:, None], atol=1e-10)


def test_cholqr_rank_deficient_drops_dependent_columns():
    rng = np.random.default_rng(2)
    B = rng.standard_normal((60, 3))
    Y = np.column_stack([B[:, 0], B[:, 1], B[:, 0] + B[:, 1], B[:, 2], 2 * B[:, 2]])
    Q, R, dropped = linalg.cholqr(Y)
    assert list(dropped) == [False, False, True, False, True]
    kept = ~dropped
    assert np.allclose(Q[:, kept].T @ Q[:, kept], np.eye(3), atol=1e-10)
    assert np.allclose(Q[:, ~kept], 0)
    assert np.allclose(Q @ R, Y, atol=1e-8)
    assert np.allclose(Y @ linalg.pinv_upper(R, dropped), Q, atol=1e-8)
    Qz, Rz, dz = linalg.cholqr(np.zeros((10, 4)))
    assert dz.all() and not Qz.any() and not Rz.any()


def _check_svd(A):
    U, s, V = linalg.jacobi_svd(A)
    s_ref = np.linalg.svd(A, compute_uv=False)
    assert np.allclose(s, s_ref, rtol=1e-12, atol=1e-12 * max(1.0, s_ref[0]))
    assert np.allclose(A @ V, U * s[None, :], atol=1e-11 * max(1.0, s_ref[0]))
    assert np.allclose(V.T @ V, np.eye(A.shape[1]), atol=1e-12)
    nz = s > 1e-12 * max(1.0, s_ref[0])
    assert np.allclose(U[:, nz].T @ U[:, nz], np.eye(nz.sum()), atol=1e-11)
    return U, s, V


def test_jacobi_against_numpy_random_sizes():
    rng = np.random.default_rng(3)
    for n in (2, 3, 5, 8, 13, 20, 33, 64, 72):
        _check_svd(rng.standard_normal((n, n)))
    _check_svd(np.triu(rng.standard_normal((72, 72))))
    _check_svd(rng.standard_normal((90, 16)))


def test_jacobi_subspaces_match_numpy():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((30, 30)) @ np.diag(np.geomspace(1e3, 1e-3, 30)) @ rng.standard_normal((30, 30))
    U, s, V = linalg.jacobi_svd(A)
    _, _, Vt = np.linalg.svd(A)
    for k in (1, 5, 10):
        cos = linalg.principal_cosines(V[:, :k], Vt[:k].T)
        assert cos.min() > 1 - 1e-9


def test_jacobi_special_matrices():
    U, s, V = linalg.jacobi_svd(np.diag([3.0, -7.0, 0.5, 0.0]))
    assert np.allclose(s, [7, 3, 0.5, 0])
    Q1, _ = np.linalg.qr(np.random.default_rng(5).standard_normal((12, 12)))
    Q2, _ = np.linalg.qr(np.random.default_rng(6).standard_normal((12, 12)))
    A = Q1 @ np.diag([5, 5, 5, 2, 2, 1, 1, 1, 1, 0, 0, 0.0]) @ Q2.T
    _check_svd(A)
    U0, s0, V0 = linalg.jacobi_svd(np.zeros((6, 6)))
    assert not s0.any() and not U0.any() and np.allclose(V0, np.eye(6))
