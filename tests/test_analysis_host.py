"""Host-side math of the analysis module (no GPU): principal cosines and the
per-singular-direction errors, against closed forms."""

import numpy as np


def _orth(rng, n, k):
    Q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return Q


def test_principal_cosines_closed_forms(metis_lib):
    from spectral_quantized_gemm_b200.analysis import principal_cosines
    rng = np.random.default_rng(0)
    V = _orth(rng, 50, 6)
    R = _orth(rng, 6, 6)                      # a rotation within the span
    assert np.allclose(principal_cosines(V, V @ R), 1.0)
    W = _orth(rng, 50, 12)
    A, B = W[:, :6], W[:, 6:]                 # orthogonal spans
    assert np.allclose(principal_cosines(A, B), 0.0, atol=1e-12)
    # planes at known angles: span(e1 cos t + e3 sin t, e2) vs span(e1, e2)
    t = 0.3
    E = np.eye(5)
    C = np.stack([np.cos(t) * E[0] + np.sin(t) * E[2], E[1]], axis=1)
    assert np.allclose(sorted(principal_cosines(C, E[:, :2])), [np.cos(t), 1.0])


def test_direction_errors_closed_forms(metis_lib):
    from spectral_quantized_gemm_b200.analysis import direction_errors
    rng = np.random.default_rng(1)
    U, V = _orth(rng, 40, 8), _orth(rng, 30, 8)
    S = np.array([9.0, 7.0, 5.0, 4.0, 3.0, 2.0, 1.0, 0.5])
    M = (U * S) @ V.T
    sig, err, leak = direction_errors(M, M)
    assert np.allclose(sig[:8], S) and np.allclose(err[:8], 0.0) and np.allclose(leak[:8], 0.0)
    eps, j = 0.25, 5
    hat = M + eps * np.outer(U[:, j], V[:, j])      # error only along direction j
    sig, err, leak = direction_errors(M, hat, n_dirs=8)
    want = np.zeros(8)
    want[j] = eps / S[j]
    assert np.allclose(err, want, atol=1e-12) and np.allclose(leak, want, atol=1e-12)
    # an error orthogonal to u_j but not to v_j shows in the leakage only
    w = _orth(rng, 40, 9)[:, 8]
    w -= U @ (U.T @ w)
    w /= np.linalg.norm(w)
    hat = M + eps * np.outer(w, V[:, j])
    sig, err, leak = direction_errors(M, hat, n_dirs=8)
    assert np.allclose(err, 0.0, atol=1e-12)
    assert np.isclose(leak[j], eps / S[j]) and np.allclose(np.delete(leak, j), 0.0, atol=1e-12)
