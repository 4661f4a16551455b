"""Pins for the oracle's randomized spectral decomposition."""

import numpy as np
import pytest

from oracle import decompose, linalg, philox
from workloads import synth


def test_sample_rows_distinct_sorted_and_uniform():
    rows, l_k = 64, 8
    counts = np.zeros(rows)
    for seed in range(2000):
        idx = decompose.sample_rows(rows, l_k, seed, 0, 0)
        assert len(idx) == l_k and len(np.unique(idx)) == l_k
        assert np.all(np.diff(idx) > 0) and idx[0] >= 0 and idx[-1] < rows
        counts[idx] += 1
    expected = 2000 * l_k / rows
    chi2 = np.sum((counts - expected) ** 2 / expected)
    assert chi2 < 120          # 63 dof
    assert list(decompose.sample_rows(10, 10, 1, 0, 0)) == list(range(10))


def test_sample_rows_is_the_smallest_keys():
    rows, l_k = 100, 7
    words = philox.element_words(3, philox.tag(2, philox.PURPOSE_SAMPLE), 5, rows)
    keys = sorted((int(w), i) for i, w in enumerate(words))
    want = sorted(i for _, i in keys[:l_k])
    assert list(decompose.sample_rows(rows, l_k, 3, 2, 5)) == want


def test_omega_box_muller_structure_and_moments():
    Om = decompose.omega(500, 72, 9, 1, 0)
    assert Om.shape == (500, 72) and Om.dtype == np.float32
    flat = Om.reshape(-1).astype(np.float64)
    assert abs(flat.mean()) < 0.01 and abs(flat.var() - 1) < 0.02
    w = philox.stream_words(9, philox.tag(1, philox.PURPOSE_OMEGA), 0, np.arange(4, dtype=np.uint64))
    u1 = (w[:, 0].astype(np.float64) + 1) * 2.0 ** -32
    r2 = flat[0:16:4] ** 2 + flat[1:16:4] ** 2
    assert np.allclose(r2, -2 * np.log(u1), rtol=1e-6)


def test_box_muller_at_the_extreme_words():
    """u1 = (a + 1) 2^-32: the largest word gives u1 = 1 (radius exactly 0) and the
    smallest u1 = 2^-32 (radius sqrt(64 ln 2), finite).  Without the +1 the word 0
    would give log(0) and the largest word a small nonzero radius, so both ends pin it.
    The angle u2 = b 2^-32: b = 0 puts the whole radius on the first draw, b = 2^30
    (a quarter turn) on the second."""
    z0, z1 = decompose.box_muller(np.array([0xFFFFFFFF, 0xFFFFFFFF]), np.array([0, 0x40000000]))
    assert np.all(z0 == 0.0) and np.all(z1 == 0.0)
    z0, z1 = decompose.box_muller(np.array([0, 0]), np.array([0, 0x40000000]))
    rad = np.sqrt(64.0 * np.log(2.0))
    assert np.all(np.isfinite(z0)) and np.all(np.isfinite(z1))
    assert z0[0] == rad and z1[0] == 0.0
    assert abs(z0[1]) < 1e-15 * rad and abs(z1[1] - rad) < 1e-15 * rad
    # the half turn b = 2^31 flips the sign of the first draw
    z0, z1 = decompose.box_muller(np.array([0]), np.array([0x80000000]))
    assert z0[0] == -rad and abs(z1[0]) < 1e-15 * rad


def test_omega_takes_box_muller_of_its_counter_words_in_pairs():
    """Element 4t, 4t+1 of Omega (row-major) come from words (w0, w1) of counter t,
    elements 4t+2, 4t+3 from (w2, w3), each draw rounded to fp32."""
    Om = decompose.omega(3, 8, 5, 2, 7).reshape(-1)
    w = philox.stream_words(5, philox.tag(2, philox.PURPOSE_OMEGA), 7, np.arange(6, dtype=np.uint64))
    for t in range(6):
        a0, a1 = decompose.box_muller(w[t, 0], w[t, 1])
        b0, b1 = decompose.box_muller(w[t, 2], w[t, 3])
        assert list(Om[4 * t:4 * t + 4]) == [np.float32(a0), np.float32(a1), np.float32(b0), np.float32(b1)]


def _planted(r, c, k, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((r, k)) @ (np.geomspace(100, 10, k)[:, None] * rng.standard_normal((k, c)))


def test_planted_rank_k_recovered_exactly():
    for (r, c, k, s, l_k) in ((64, 48, 4, 4, 16), (128, 96, 6, 2, 128)):
        M = _planted(r, c, k, 7)
        out = decompose.refresh_basis(M, k, s, l_k, 1, 0, 0)
        _, _, Vt = np.linalg.svd(M)
        cos = linalg.principal_cosines(out["V"], Vt[:k].T)
        assert cos.min() > 1 - 1e-10
        U, S, V = decompose.step_factors(M, out["V"])
        resid = M - (U * S) @ V.T
        assert np.linalg.norm(resid) / np.linalg.norm(M) < 1e-12
        assert np.allclose(S, np.linalg.svd(M, compute_uv=False)[:k], rtol=1e-10)


def test_step_factors_is_the_projection_and_orthonormal():
    rng = np.random.default_rng(8)
    M = rng.standard_normal((80, 40))
    V0, _ = np.linalg.qr(rng.standard_normal((40, 6)))
    U, S, V = decompose.step_factors(M, V0)
    assert np.allclose((U * S) @ V.T, M @ V0 @ V0.T, atol=1e-10)
    assert np.allclose(U.T @ U, np.eye(6), atol=1e-10)
    assert np.allclose(V.T @ V, np.eye(6), atol=1e-10)
    assert np.all(np.diff(S) <= 0)
    for j in range(6):
        assert V[np.argmax(np.abs(V[:, j])), j] > 0
    R = decompose.residual(M, U, S, V)
    assert R.dtype == np.float32
    assert np.allclose(R.astype(np.float64) + (U * S) @ V.T, M, atol=1e-5)


def test_zero_matrix_gives_empty_factors():
    M = np.zeros((64, 32))
    out = decompose.refresh_basis(M, 4, 4, 16, 0, 0, 0)
    assert not out["V"].any()
    U, S, V = decompose.step_factors(M, np.eye(32)[:, :4])
    assert not S.any() and not U.any()
    assert not decompose.residual(M, U, S, V).any()


def test_tiny_workload_residual_spectrum():
    """关键设计 1 / 消融: the residual spectrum is flat once the spikes are absorbed.

    Tiny workload (6 spikes 640 * 0.8^i over an N(0,1) bulk whose edge is
    sqrt(256) + sqrt(256) = 32): with an unsampled sketch and k = 4 the residual
    keeps exactly the 5th and 6th singular values of X, the rest lie at the
    bulk edge; with k = 6 nothing is left above the edge.
    """
    cfg = synth.CONFIGS["tiny_fwd"]
    X = synth.operand_matrix(cfg, "X", as_numpy=True)
    sx = np.linalg.svd(X, compute_uv=False)
    edge = 32.0
    out = decompose.refresh_basis(X, 4, 4, 256, cfg["seed"], 0, 0)
    U, S, V = decompose.step_factors(X, out["V"])
    sr = np.linalg.svd(decompose.residual(X, U, S, V).astype(np.float64), compute_uv=False)
    assert np.allclose(sr[:2], sx[4:6], rtol=0.02)
    assert sr[2] < 1.1 * edge
    out6 = decompose.refresh_basis(X, 6, 4, 256, cfg["seed"], 0, 0)
    U6, S6, V6 = decompose.step_factors(X, out6["V"])
    sr6 = np.linalg.svd(decompose.residual(X, U6, S6, V6).astype(np.float64), compute_uv=False)
    assert sr6[0] < 1.1 * edge
    # sampled sketch (l_k = 32 of 256 rows): the residual is still far narrower than X
    outs = decompose.refresh_basis(X, 4, 4, 32, cfg["seed"], 0, 0)
    Us, Ss, Vs = decompose.step_factors(X, outs["V"])
    srs = np.linalg.svd(decompose.residual(X, Us, Ss, Vs).astype(np.float64), compute_uv=False)
    assert srs[0] < 0.6 * sx[0]
    assert np.abs(decompose.residual(X, U6, S6, V6)).max() < 0.5 * np.abs(X).max()


def test_refresh_argument_checks():
    with pytest.raises(ValueError):
        decompose.refresh_basis(np.zeros((16, 16)), 4, 8, 8, 0, 0, 0)
    with pytest.raises(ValueError):
        decompose.sample_rows(10, 0, 0, 0, 0)
