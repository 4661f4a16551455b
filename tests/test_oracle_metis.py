"""Pins for the oracle's Metis product and layer."""

import numpy as np

from oracle import decompose, formats, metis, nvfp4, philox
from workloads import synth


def _grid_matrix(rows, cols, rng):
    """Every 16-block holds E2M1 grid values with block max 6 times a power of two."""
    mags = formats.E2M1_MAGNITUDES
    v = mags[rng.integers(0, 8, size=(rows, cols))] * rng.choice([-1.0, 1.0], size=(rows, cols))
    v[:, ::16] = 6.0
    v[::16, :] = 6.0
    return v


def test_k0_is_plain_nvfp4_and_lossless_on_grid_inputs():
    """k = 0 reduces to plain NVFP4 GeMM; on inputs whose 16-blocks in both
    orientations are exactly representable the product is the exact X W."""
    rng = np.random.default_rng(0)
    X = _grid_matrix(64, 96, rng)
    W = _grid_matrix(96, 48, rng)
    D = _grid_matrix(64, 48, rng)
    ops = [metis.prepare_operand(M, None) for M in (X, W, D)]
    assert np.array_equal(metis.linear_fwd(ops[0], ops[1]), X @ W)
    dX, dW = metis.linear_bwd(*ops)
    assert np.array_equal(dX, D @ W.T) and np.array_equal(dW, X.T @ D)


def test_identity_quantizer_reproduces_exact_product():
    """With Q replaced by the identity the split is exact: hat(M) == M."""
    cfg = synth.CONFIGS["tiny_fwd"]
    X = synth.operand_matrix(cfg, "X", as_numpy=True)
    W = synth.operand_matrix(cfg, "W", as_numpy=True)
    hats = []
    for M, op in ((X, 0), (W, 1)):
        V = decompose.refresh_basis(M, 4, 4, 32, 0, op, 0)["V"]
        U, S, Vn = decompose.step_factors(M, V)
        R = M - (U * S) @ Vn.T                      # unrounded residual
        hats.append((U * S) @ Vn.T + R)
    Y = hats[0] @ hats[1]
    assert np.allclose(Y, X @ W, rtol=0, atol=1e-9 * np.abs(X @ W).max())


def test_fold_expansion_equals_dense_product():
    rng = np.random.default_rng(1)
    p, K, q, k = 20, 32, 24, 3
    LA, RA, AR = rng.standard_normal((p, k)), rng.standard_normal((K, k)), rng.standard_normal((p, K))
    LB, RB, BR = rng.standard_normal((K, k)), rng.standard_normal((q, k)), rng.standard_normal((K, q))
    SA, SB = rng.uniform(1, 5, k), rng.uniform(1, 5, k)
    dense = ((LA * SA) @ RA.T + AR) @ ((LB * SB) @ RB.T + BR)
    assert np.allclose(metis.fold_terms((LA, SA, RA, AR), (LB, SB, RB, BR)), dense, atol=1e-10)


def test_factor_tensor_scale_is_the_smallest_power_of_two():
    for amax in (1.0, 2688.0, 2689.0, 1e-3, 5.0e-40 + 1e-30):
        F = np.array([[amax]], dtype=np.float32)
        g = metis.factor_tensor_scale(F)
        assert g == 2.0 ** np.round(np.log2(g))
        assert np.float32(amax) / np.float32(2688.0) <= g
        assert np.float32(amax) / np.float32(2688.0) > g / 2
    assert metis.factor_tensor_scale(np.zeros((3, 3), dtype=np.float32)) == 1.0


def test_factor_quantization_blocks_run_along_the_long_dimension():
    rng = np.random.default_rng(2)
    F = rng.standard_normal((64, 5)).astype(np.float32) / 8
    codes, scales, g = metis.quantize_factor(F)
    assert codes.shape == (5, 64) and scales.shape == (5, 4)
    back = nvfp4.dequantize_blocks(codes, scales, g).T
    assert np.abs(back - F).max() <= 0.25 * np.abs(F).max()


def _operand_hats(cfg, name, k, s, l_k, op_id):
    M = synth.operand_matrix(cfg, name, as_numpy=True)
    V = decompose.refresh_basis(M, k, s, l_k, 0, op_id, 0)["V"]
    metis_hat = metis.operand_hat(metis.prepare_operand(M, V, operand_id=op_id), "row")
    plain_hat = metis.operand_hat(metis.prepare_operand(M, None), "row")
    return M, metis_hat, plain_hat


def test_metis_preserves_small_singular_components():
    """研究背景 / 核心矛盾 and 关键设计 1: block quantization of an anisotropic
    matrix lets a few large values set the block scale, so small values round
    to zero and the small singular components are distorted; splitting off
    the dominant subspace before quantizing keeps them.

    On the layer-shaped workload (spikes on 2% of the hidden dimensions):
    * plain NVFP4 rounds a large share of the small entries to zero;
    * the relative error of X_hat restricted to the tail (non-spike) right
      singular subspace is clearly lower with Metis.
    (The total Frobenius error is not lower: Q_b also quantizes the dominant
    factors U and V, which costs ~10% RMS on the dominant energy.)
    """
    cfg = synth.scaled_config("gpt2_small_mlp_up", l=1024, m=768, n=768)
    X, xm, xp = _operand_hats(cfg, "X", 12, 8, 82, 0)
    small = np.abs(X) < 1.0
    assert np.mean(xp[small] == 0) > 0.15
    _, _, Vt = np.linalg.svd(X, full_matrices=False)
    T = Vt[synth.n_spikes(*X.shape):].T
    err_m = np.linalg.norm((xm - X) @ T) / np.linalg.norm(X @ T)
    err_p = np.linalg.norm((xp - X) @ T) / np.linalg.norm(X @ T)
    assert err_m < 0.75 * err_p


def test_weight_gradient_uses_the_column_wise_residual():
    """Reading R5: each GeMM reads the quantization with 16-blocks along its own
    contraction dimension.  X below is exact in column-wise blocks (16 rows of a column
    share a power-of-two scale) but lossy in row-wise blocks (columns of scale 2^6 and
    2^-6 side by side); D is exact column-wise.  So dW = X^T D exactly, while the
    row-wise quantization of X would lose its small columns."""
    rng = np.random.default_rng(7)
    l, m, n = 64, 32, 48
    mags = formats.E2M1_MAGNITUDES
    expo = np.where(np.arange(m) % 2 == 0, 6.0, -6.0)
    X = mags[rng.integers(0, 8, size=(l, m))] * rng.choice([-1.0, 1.0], size=(l, m))
    X[::16, :] = 6.0
    X = X * 2.0 ** expo[None, :]
    D = mags[rng.integers(0, 8, size=(l, n))] * rng.choice([-1.0, 1.0], size=(l, n))
    D[::16, :] = 6.0
    W = rng.standard_normal((m, n))
    ops = [metis.prepare_operand(M, None) for M in (X, W, D)]
    _, dW = metis.linear_bwd(*ops)
    assert np.array_equal(dW, X.T @ D)
    assert not np.array_equal(metis.dequant_residual(ops[0], "row"), X)   # the row-wise one is lossy


def _exact_one_way(rows, cols, rng, exact):
    """Grid values whose 16-blocks are exact in one orientation only: exact="row" gives
    every row a power-of-two scale of its own (2^6 or 2^-6, alternating), so row-wise
    blocks are exact and column-wise blocks, which mix the two, are not; exact="col"
    does the same per column."""
    mags = formats.E2M1_MAGNITUDES
    v = mags[rng.integers(0, 8, size=(rows, cols))] * rng.choice([-1.0, 1.0], size=(rows, cols))
    if exact == "row":
        v[:, ::16] = 6.0
        return v * np.where(np.arange(rows) % 2 == 0, 2.0 ** 6, 2.0 ** -6)[:, None]
    v[::16, :] = 6.0
    return v * np.where(np.arange(cols) % 2 == 0, 2.0 ** 6, 2.0 ** -6)[None, :]


def test_forward_and_input_gradient_use_their_own_orientations():
    """Reading R5 for the other two GeMMs: Y = X W reads X row-wise and W column-wise;
    dX = D W^T reads D and W row-wise.  With each operand exact only in the orientation
    its GeMM should read, both products are exact."""
    rng = np.random.default_rng(8)
    l, m, n = 64, 48, 32
    X, W = _exact_one_way(l, m, rng, "row"), _exact_one_way(m, n, rng, "col")
    ops = [metis.prepare_operand(M, None) for M in (X, W)]
    assert np.array_equal(metis.linear_fwd(*ops), X @ W)
    assert not np.array_equal(metis.dequant_residual(ops[0], "col"), X)
    assert not np.array_equal(metis.dequant_residual(ops[1], "row"), W)
    D, W2 = _exact_one_way(l, n, rng, "row"), _exact_one_way(m, n, rng, "row")
    ops = [metis.prepare_operand(M, None) for M in (X, W2, D)]
    dX, _ = metis.linear_bwd(*ops)
    assert np.array_equal(dX, D @ W2.T)
    assert not np.array_equal(metis.dequant_residual(ops[2], "col"), D)


def test_factor_sr_sub_streams_by_hand():
    """Which stochastic-rounding stream each factor draws (reading R4: U from sub-stream 2,
    V from sub-stream 3 of the operand's SR purpose), worked by hand on a 16 x 16 factor.

    Every block (a column of F: blocks run along the long dimension) has maximum 6, so
    g = 2^-8 (the smallest power of two with 6 <= 2688 g), the block scale is E4M3(256) =
    256 and the scaled values are F itself.  All other entries sit at midpoints of the
    E2M1 grid (p = 1/2), where the rule rounds up iff the element's 16-bit field is at
    least 2^15: its top bit.  The expected codes follow from the fields alone."""
    rng = np.random.default_rng(11)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    lo_idx = np.array([0, 1, 2, 3, 4, 5, 6])          # index of the grid point below each midpoint
    pick = rng.integers(0, 7, size=(16, 16))
    sign = rng.choice([-1.0, 1.0], size=(16, 16))
    F = (mids[pick] * sign).astype(np.float32)
    F[0, :] = 6.0
    pick[0, :] = -1
    seed, op_id, step = 21, 4, 9
    for sub in (philox.SR_SUB_LEFT, philox.SR_SUB_RIGHT):
        codes, scales, g = metis.quantize_factor(F, seed, op_id, sub, step, "sr")
        assert g == 2.0 ** -8 and np.all(scales == formats.e4m3_encode_rn(np.array([256.0]))[0])
        fields = philox.sr_fields(seed, op_id, sub, step, 256).reshape(16, 16)   # k x long view
        want = np.empty((16, 16), dtype=np.uint8)
        for i in range(16):              # column i of F = row i of the transposed view
            for j in range(16):          # row j of F = element j of the block
                if pick[j, i] < 0:
                    want[i, j] = 7
                else:
                    want[i, j] = lo_idx[pick[j, i]] + (fields[i, j] >> 15)
                want[i, j] |= np.uint8(8) if sign[j, i] < 0 and pick[j, i] >= 0 else np.uint8(0)
        assert np.array_equal(codes, want), sub
    left = metis.quantize_factor(F, seed, op_id, philox.SR_SUB_LEFT, step, "sr")[0]
    right = metis.quantize_factor(F, seed, op_id, philox.SR_SUB_RIGHT, step, "sr")[0]
    assert np.mean(left != right) > 0.3                 # the two streams are distinct draws


def test_prepare_operand_draws_u_from_left_and_v_from_right():
    """prepare_operand quantizes U with sub-stream 2 and V with sub-stream 3 (the
    convention the test above works by hand), not the other way round."""
    M = synth.operand_matrix(synth.CONFIGS["tiny_fwd"], "X", as_numpy=True)
    V = decompose.refresh_basis(M, 4, 4, 32, 0, 0, 0)["V"]
    op = metis.prepare_operand(M, V, seed=5, operand_id=0, step=3, rounding="sr")
    U32, V32 = op["U"].astype(np.float32), op["V"].astype(np.float32)
    for F, q, own, other in ((U32, op["Uq"], philox.SR_SUB_LEFT, philox.SR_SUB_RIGHT),
                             (V32, op["Vq"], philox.SR_SUB_RIGHT, philox.SR_SUB_LEFT)):
        assert np.array_equal(q[0], metis.quantize_factor(F, 5, 0, own, 3, "sr")[0])
        assert not np.array_equal(q[0], metis.quantize_factor(F, 5, 0, other, 3, "sr")[0])
