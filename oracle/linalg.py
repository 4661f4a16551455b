"""CholQR and one-sided Jacobi SVD in fp64.

The Metis notes ("Metis: Training LLMs with FP4 Quantization", 关键设计 2)
recover the dominant subspace by randomized SVD of a sampled sketch; they
name a "customized low-rank spectral decomposition operator" (关键设计 3) but
give no algorithm for its small dense steps.  The build's plainest reading
uses the two textbook routines below.

CholQR (Cholesky QR): for a tall Y (m x n, m >= n), G = Y^T Y, R = chol(G)
upper-triangular with G = R^T R, Q = Y R^{-1}.  Reading for rank-deficient
input: a pivot d_j = G_jj - sum_{i<j} R_ij^2 that is not above
DROP_TOL * max_i G_ii marks column j as linearly dependent on the earlier
ones; row j of R and column j of Q are then set to zero (so Q R reproduces Y
up to the dropped, numerically null, components).

One-sided (Hestenes) Jacobi SVD: columns p < q of A are rotated in cyclic
order until every pair satisfies |a_p . a_q| <= tol * |a_p| |a_q| (tol 1e-12: at 1e-15 fp64
rounding noise of length-64 dot products keeps pairs above the bound);
the accumulated rotations are V, the column norms are the singular values and
the normalised columns are U.

Pins (tests/test_oracle_linalg.py): Q^T Q = I and Q R = Y on random and
rank-deficient inputs; Jacobi singular values and subspaces against
numpy.linalg.svd on random matrices of sizes 2..72, on matrices with
repeated and zero singular values, and on diagonal matrices.
"""

import numpy as np

DROP_TOL = 1e-12
JACOBI_TOL = 1e-12
JACOBI_MAX_SWEEPS = 60


def cholqr(Y):
    """Returns (Q, R, dropped) for Y (m x n) in fp64."""
    Y = np.asarray(Y, dtype=np.float64)
    m, n = Y.shape
    G = Y.T @ Y
    R = np.zeros((n, n))
    dropped = np.zeros(n, dtype=bool)
    gmax = max(float(np.max(np.diag(G))), 0.0) if n else 0.0
    tol = DROP_TOL * gmax
    for j in range(n):
        d = G[j, j] - np.dot(R[:j, j], R[:j, j])
        if not (d > tol) or gmax == 0.0:
            dropped[j] = True
            continue
        R[j, j] = np.sqrt(d)
        for t in range(j + 1, n):
            R[j, t] = (G[j, t] - np.dot(R[:j, j], R[:j, t])) / R[j, j]
    Q = np.zeros((m, n))
    for j in range(n):
        if dropped[j]:
            continue
        v = Y[:, j] - Q[:, :j] @ R[:j, j]
        Q[:, j] = v / R[j, j]
    return Q, R, dropped


def pinv_upper(R, dropped):
    """Inverse of upper-triangular R on its kept rows/columns, zero elsewhere.

    Satisfies Y pinv_upper(R) == Q for (Q, R, dropped) = cholqr(Y).
    """
    n = R.shape[0]
    Rinv = np.zeros((n, n))
    for j in range(n):
        if dropped[j]:
            continue
        # column j of R^{-1}: solve R x = e_j restricted to kept indices
        x = np.zeros(n)
        x[j] = 1.0 / R[j, j]
        for i in range(j - 1, -1, -1):
            if dropped[i]:
                continue
            x[i] = -np.dot(R[i, i + 1:j + 1], x[i + 1:j + 1]) / R[i, i]
        Rinv[:, j] = x
    return Rinv


def jacobi_svd(A, tol=JACOBI_TOL, max_sweeps=JACOBI_MAX_SWEEPS):
    """One-sided Jacobi SVD of A (m x n, m >= n): returns (U, sigma, V).

    A V = U diag(sigma); sigma descending; zero singular values give zero
    columns of U.
    """
    U = np.array(A, dtype=np.float64, copy=True)
    m, n = U.shape
    V = np.eye(n)
    sweeps = 0
    for sweeps in range(1, max_sweeps + 1):
        rotated = False
        for p in range(n - 1):
            for q in range(p + 1, n):
                alpha = np.dot(U[:, p], U[:, p])
                beta = np.dot(U[:, q], U[:, q])
                gamma = np.dot(U[:, p], U[:, q])
                if gamma == 0.0 or abs(gamma) <= tol * np.sqrt(alpha * beta):
                    continue
                rotated = True
                zeta = (beta - alpha) / (2.0 * gamma)
                t = (1.0 if zeta >= 0 else -1.0) / (abs(zeta) + np.hypot(1.0, zeta))
                c = 1.0 / np.sqrt(1.0 + t * t)
                s = c * t
                up = U[:, p].copy()
                U[:, p] = c * up - s * U[:, q]
                U[:, q] = s * up + c * U[:, q]
                vp = V[:, p].copy()
                V[:, p] = c * vp - s * V[:, q]
                V[:, q] = s * vp + c * V[:, q]
        if not rotated:
            break
    else:
        raise RuntimeError("Jacobi SVD did not converge")
    sigma = np.sqrt(np.sum(U * U, axis=0))
    order = np.argsort(-sigma, kind="stable")
    sigma = sigma[order]
    U = U[:, order]
    V = V[:, order]
    nz = sigma > 0
    U[:, nz] = U[:, nz] / sigma[nz]
    U[:, ~nz] = 0.0
    return U, sigma, V


def principal_cosines(A, B):
    """Cosines of the principal angles between span(A) and span(B), descending."""
    qa, _ = np.linalg.qr(np.asarray(A, dtype=np.float64))
    qb, _ = np.linalg.qr(np.asarray(B, dtype=np.float64))
    return np.clip(np.linalg.svd(qa.T @ qb, compute_uv=False), 0.0, 1.0)
