"""Pins for the oracle's LoRA-SVD linear projection (W = W_res + beta L2 L1)."""

import numpy as np
import torch

from oracle import formats, lora_svd, nvfp4


def test_bf16_round_matches_torch_and_ties_go_even():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(4096) * 10.0 ** rng.uniform(-20, 20, 4096)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(lora_svd.bf16_round(x), want)
    # exact halves between two bf16 neighbours: the even one (lowest kept bit 0) wins
    assert lora_svd.bf16_round(np.float32(1.0 + 2.0 ** -8)) == 1.0                    # 1.0 is even
    assert lora_svd.bf16_round(np.float32(1.0 + 3 * 2.0 ** -8)) == 1.0 + 2.0 ** -6    # 1 + 2^-7 is odd
    assert lora_svd.bf16_round(np.float32(-(1.0 + 2.0 ** -9))) == -1.0
    assert lora_svd.bf16_round(np.float32(1.0 + 2.0 ** -8 + 2.0 ** -20)) == 1.0 + 2.0 ** -7


def _random_nvfp4(outer, inner, rng):
    codes = rng.integers(0, 16, size=(outer, inner)).astype(np.uint8)
    scales = formats.e4m3_encode_rn(2.0 ** rng.integers(-3, 3, size=(outer, inner // 16)))
    return nvfp4.dequantize_blocks(codes, scales, 0.5)


def test_beta_zero_is_the_plain_nvfp4_gemm():
    """beta = 0: the branch vanishes and the product is the decoded FP4 GeMM, here
    summed element by element in Python."""
    rng = np.random.default_rng(1)
    p, K, q, k = 3, 32, 4, 2
    A, B = _random_nvfp4(p, K, rng), _random_nvfp4(q, K, rng)
    M = rng.standard_normal((p, K))
    L2, L1 = rng.standard_normal((K, k)), rng.standard_normal((k, q))
    C, _ = lora_svd.lora_linear(0, A, B, M, L2, L1, 0.0)
    for i in range(p):
        for j in range(q):
            s = 0.0
            for x in range(K):
                s += A[i, x] * B[j, x]
            assert abs(C[i, j] - s) <= 1e-12 * max(1.0, abs(s))


def test_rank1_all_ones_branch_gives_row_sums():
    """A = B = 0, k = 1, L2 and L1 all ones: every output entry is beta times the row
    sum of M, in both orientations; 1 + 2^-9 rounds to 1 in bf16, so it acts as 1."""
    rng = np.random.default_rng(2)
    p, K, q, beta = 5, 64, 7, 0.75
    M = rng.standard_normal((p, K))
    rs = M.sum(axis=1)
    one = 1.0 + 2.0 ** -9
    C0, T0 = lora_svd.lora_linear(0, np.zeros((p, K)), np.zeros((q, K)), M, np.full((K, 1), one),
                                  np.full((1, q), one), beta)
    C1, T1 = lora_svd.lora_linear(1, np.zeros((p, K)), np.zeros((q, K)), M, np.full((q, 1), one),
                                  np.full((1, K), one), beta)
    for C, T in ((C0, T0), (C1, T1)):
        assert np.allclose(T[:, 0], rs, rtol=0, atol=1e-12)
        assert np.allclose(C, beta * rs[:, None] * np.ones((1, q)), rtol=0, atol=1e-12)


def _grid(shape, rng, lo=-8, hi=8, unit=2.0 ** -4):
    """Small multiples of 2^-4: exactly representable in bf16, also after a step of 2^-4."""
    return rng.integers(lo, hi, size=shape) * unit


def test_gradients_are_finite_differences_of_the_forward():
    """On bf16-exact factors (so the bf16 casts are exact), with the FP4 operands held
    fixed: dL2 = branch_grad(X, T of which = 1), dL1 = branch_grad(D, T of which = 0)^T
    and dX = lora_linear(which = 1) are the central differences of <D, Y>, Y the
    forward product; the forward is bilinear, so the differences are exact."""
    rng = np.random.default_rng(3)
    l, m, n, k, beta = 6, 5, 4, 3, 0.5
    X, D = rng.standard_normal((l, m)), rng.standard_normal((l, n))
    W_hat = rng.standard_normal((m, n))          # stands for the decoded Q(W_res)
    L2, L1 = _grid((m, k), rng), _grid((k, n), rng)
    h = 2.0 ** -4

    def loss(X_, L2_, L1_):
        Y, _ = lora_svd.lora_linear(0, X_, W_hat.T, X_, L2_, L1_, beta)
        return float(np.sum(D * Y))

    _, T_x = lora_svd.lora_linear(0, X, W_hat.T, X, L2, L1, beta)
    dX, T_d = lora_svd.lora_linear(1, D, W_hat, D, L2, L1, beta)
    dL2 = lora_svd.branch_grad(X, T_d, beta)
    dL1 = lora_svd.branch_grad(D, T_x, beta).T
    for (i, j) in np.ndindex(m, k):
        E = np.zeros_like(L2)
        E[i, j] = h
        fd = (loss(X, L2 + E, L1) - loss(X, L2 - E, L1)) / (2 * h)
        assert abs(fd - dL2[i, j]) <= 1e-9 * max(1.0, abs(fd))
    for (i, j) in np.ndindex(k, n):
        E = np.zeros_like(L1)
        E[i, j] = h
        fd = (loss(X, L2, L1 + E) - loss(X, L2, L1 - E)) / (2 * h)
        assert abs(fd - dL1[i, j]) <= 1e-9 * max(1.0, abs(fd))
    for (i, j) in np.ndindex(l, m):
        E = np.zeros_like(X)
        E[i, j] = h
        fd = (loss(X + E, L2, L1) - loss(X - E, L2, L1)) / (2 * h)
        assert abs(fd - dX[i, j]) <= 1e-9 * max(1.0, abs(fd))


def test_constraint_is_qr_and_keeps_the_product():
    rng = np.random.default_rng(4)
    m, n, k = 40, 24, 6
    L2, L1 = rng.standard_normal((m, k)), rng.standard_normal((k, n))
    Q, L1n = lora_svd.constrain(L2, L1)
    assert np.allclose(Q.T @ Q, np.eye(k), atol=1e-12)
    assert np.allclose(Q @ L1n, L2 @ L1, atol=1e-12)
    Qn, Rn = np.linalg.qr(L2)
    sgn = np.sign(np.diag(Rn))
    assert np.allclose(Q, Qn * sgn[None, :], atol=1e-12)
    assert np.allclose(L1n, (Rn * sgn[:, None]) @ L1, atol=1e-12)
    # a dependent column is dropped and the product still holds
    L2d = L2.copy()
    L2d[:, 3] = 2.0 * L2d[:, 1] - L2d[:, 0]
    Qd, L1d = lora_svd.constrain(L2d, L1)
    assert np.allclose(Qd[:, 3], 0.0)
    assert np.allclose(Qd @ L1d, L2d @ L1, atol=1e-10)


def test_realign_keeps_w_and_recovers_an_exact_rank_k_split():
    rng = np.random.default_rng(5)
    m, n, k, s, beta = 64, 48, 4, 4, 0.5
    # W_eff of exact rank k with well separated singular values, all in the branch
    U0, _ = np.linalg.qr(rng.standard_normal((m, k)))
    V0, _ = np.linalg.qr(rng.standard_normal((n, k)))
    S0 = np.array([40.0, 20.0, 10.0, 5.0])
    W_res = np.zeros((m, n))
    L2, L1 = U0 @ np.diag(S0), V0.T / beta
    W_eff = W_res + beta * L2 @ L1
    Wn, L2n, L1n, S = lora_svd.realign(W_res, L2, L1, beta, k, s, seed=7, operand_id=1, step=0)
    assert np.allclose(Wn + beta * L2n @ L1n, W_eff, atol=1e-12)
    assert np.allclose(L2n.T @ L2n, np.eye(k), atol=1e-10)
    # bf16 rounding of W_eff (relative 2^-9) bounds what the rank-k part misses
    assert np.linalg.norm(Wn) <= 4e-3 * np.linalg.norm(W_eff)
    assert np.allclose(S, np.linalg.svd(W_eff, compute_uv=False)[:k], rtol=4e-3)
    # W_res carrying a noise floor: the branch takes the top-k directions
    noise = 0.01 * rng.standard_normal((m, n))
    Wn2, L2n2, L1n2, S2 = lora_svd.realign(noise, L2, L1, beta, k, s, seed=7, operand_id=1, step=0)
    assert np.allclose(Wn2 + beta * L2n2 @ L1n2, noise + W_eff, atol=1e-12)
    assert np.allclose(S2, np.linalg.svd(noise + W_eff, compute_uv=False)[:k], rtol=1e-2)


def test_realign_decomposes_the_bf16_copy():
    """A constant W_eff = c (c = 1 + 2^-8 + 2^-10, not a bf16 number; bf16(c) = 1 + 2^-7):
    the decomposition sees bf16(W_eff), a rank-1 matrix with singular value
    bf16(c) sqrt(m n), and the new residual is exactly the rounding c - bf16(c)."""
    m, n, beta = 64, 48, 2.0
    c = 1.0 + 2.0 ** -8 + 2.0 ** -10
    cb = 1.0 + 2.0 ** -7
    assert lora_svd.bf16_round(np.float32(c)) == cb
    W_res = np.full((m, n), c)
    Wn, L2n, L1n, S = lora_svd.realign(W_res, np.zeros((m, 1)), np.zeros((1, n)), beta, 1, 4, seed=3,
                                       operand_id=1, step=0)
    assert abs(S[0] - cb * np.sqrt(m * n)) <= 1e-12 * S[0]
    assert np.allclose(Wn, c - cb, rtol=0, atol=1e-12)
    assert np.allclose(beta * L2n @ L1n, cb, rtol=0, atol=1e-12)
