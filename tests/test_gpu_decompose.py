"""GPU randomized decomposition vs the oracle.

Contract: identical sampled rows, the same Gaussian test matrix
(within 1 fp32 ulp: both sides evaluate Box-Muller in fp64), and subspace
cosines >= 0.999 for the recovered basis and factors.  Factor quantization is
bit-exact given the GPU's own fp32 factors.
"""

import numpy as np
import pytest
import torch

from oracle import decompose, linalg, metis, philox
from tests.gpu_helpers import codes_unpacked
from workloads import synth

pytestmark = pytest.mark.gpu
COS = 0.999


def _gpu_decompose(ctx, M, k, s, l_k, seed, op, refresh=True, step=0, factors=None, rounding=0):
    rows, cols = M.shape
    f = factors or ctx.new_factors(rows, cols, k, s, l_k, keep_sketch=True)
    ctx.decompose(M, k=k, s=s, l_k=l_k, seed=seed, operand_id=op, refresh=refresh, step=step, factors=f,
                  rounding=rounding)
    torch.cuda.synchronize()
    return f


def _compare(ctx, cfg, name, k, s, l_k, op, seed):
    Mt = synth.operand_matrix(cfg, name)
    M = Mt.double().numpy()
    f = _gpu_decompose(ctx, Mt.cuda(), k, s, l_k, seed, op)
    assert ctx.poll_device_status() == 0
    ref = decompose.refresh_basis(M, k, s, l_k, seed, op, 0)
    assert np.array_equal(f.sampled_rows.cpu().numpy()[:l_k], ref["rows"])
    om = f.omega.cpu().numpy()
    ulp = np.spacing(np.abs(ref["omega"]).astype(np.float32))
    assert np.all(np.abs(om - ref["omega"]) <= ulp)
    U, S, V = decompose.step_factors(M, ref["V"])
    gV, gU, gS = f.V.cpu().double().numpy(), f.U.cpu().double().numpy(), f.S.cpu().double().numpy()[:k]
    assert linalg.principal_cosines(gV, V).min() >= COS
    assert linalg.principal_cosines(gU, U).min() >= COS
    assert np.max(np.abs(gS - S) / S[0]) < 1e-3
    assert np.all(np.diff(gS) <= 1e-6 * gS[0])
    assert np.allclose(gV.T @ gV, np.eye(k), atol=1e-4)
    assert np.allclose(gU.T @ gU, np.eye(k), atol=1e-3)
    for j in range(k):                        # sign convention
        assert gV[np.argmax(np.abs(gV[:, j])), j] > 0
    # the split reproduces the projection of M onto the basis
    low = (gU * gS) @ gV.T
    proj = M @ gV @ gV.T
    assert np.linalg.norm(low - proj) / np.linalg.norm(proj) < 1e-4
    return f, M


def test_tiny_workload(ctx, metis_lib):
    cfg = synth.CONFIGS["tiny_fwd"]
    _compare(ctx, cfg, "X", 4, 4, 32, 0, 0)
    _compare(ctx, cfg, "W", 4, 4, 256, 1, 0)


def test_gpt2_shapes(ctx, metis_lib):
    cfg = synth.CONFIGS["gpt2_small_mlp_up"]
    _compare(ctx, cfg, "X", 12, 8, 82, 0, 1)
    _compare(ctx, cfg, "W", 12, 8, 768, 1, 1)


def test_llama_x_and_wide_sketch(ctx, metis_lib):
    cfg = synth.CONFIGS["llama3_8b_mlp_up"]
    _compare(ctx, cfg, "X", 64, 8, 82, 0, 2)
    # widest supported sketch (k + s = 128) on a smaller matrix
    cfg2 = synth.scaled_config("llama3_8b_mlp_up", l=1024, m=1024, n=1024)
    _compare(ctx, cfg2, "X", 64, 64, 256, 0, 2)


def test_reuse_keeps_the_span(ctx, metis_lib):
    cfg = synth.CONFIGS["gpt2_small_mlp_up"]
    Mt = synth.operand_matrix(cfg, "X")
    f = _gpu_decompose(ctx, Mt.cuda(), 12, 8, 82, 1, 0)
    V0 = f.V.cpu().double().numpy()
    M1 = synth.perturbed(dict(cfg, perturb=1e-2), "X", Mt, 1)
    _gpu_decompose(ctx, M1.cuda(), 12, 8, 82, 1, 0, refresh=False, step=1, factors=f)
    V1 = f.V.cpu().double().numpy()
    assert linalg.principal_cosines(V0, V1).min() > 1 - 1e-6
    U, S, V = decompose.step_factors(M1.double().numpy(), V0)
    assert np.max(np.abs(f.S.cpu().double().numpy()[:12] - S) / S[0]) < 1e-3


def test_factor_quantization_bit_exact(ctx, metis_lib):
    cfg = synth.CONFIGS["gpt2_small_mlp_up"]
    Mt = synth.operand_matrix(cfg, "X")
    f = _gpu_decompose(ctx, Mt.cuda(), 12, 8, 82, 1, 0, rounding=1, step=5)
    for fac, q, sub, n in ((f.U, f.Uq, philox.SR_SUB_LEFT, 8192), (f.V, f.Vq, philox.SR_SUB_RIGHT, 768)):
        F = fac.cpu().numpy()
        codes, scales, g = codes_unpacked(q)
        wc, ws, wg = metis.quantize_factor(F, seed=1, operand_id=0, sub=sub, step=5, rounding="sr")
        assert g == wg
        assert np.array_equal(codes[:12], wc) and np.array_equal(scales[:12], ws)
        assert not codes[12:].any() and not scales[12:].any()


def test_planted_low_rank(ctx, metis_lib):
    rng = np.random.default_rng(3)
    r, c, k = 1024, 512, 8
    M = rng.standard_normal((r, k)) @ (np.geomspace(50, 5, k)[:, None] * rng.standard_normal((k, c)))
    Mt = torch.from_numpy(M).to(torch.bfloat16)
    Mb = Mt.double().numpy()
    Us, sv, Vt = np.linalg.svd(Mb, full_matrices=False)
    best = np.sqrt(np.sum(sv[k:] ** 2))
    # sampled sketch (128 of 1024 rows): the planted subspace is recovered
    f = _gpu_decompose(ctx, Mt.cuda(), k, 4, 128, 0, 0)
    assert linalg.principal_cosines(f.V.cpu().double().numpy(), Vt[:k].T).min() > 1 - 1e-5
    # unsampled sketch: bf16 rounding of the planted matrix adds a small full-rank
    # part, and the split leaves no more than the best rank-k approximation does
    # (Eckart-Young), up to the sketch's own accuracy
    f = _gpu_decompose(ctx, Mt.cuda(), k, 4, r, 0, 0)
    low = (f.U.cpu().double().numpy() * f.S.cpu().double().numpy()[:k]) @ f.V.cpu().double().numpy().T
    assert np.linalg.norm(Mb - low) <= 1.02 * best + 1e-6 * np.linalg.norm(Mb)


def test_zero_and_nonfinite_inputs(ctx, metis_lib):
    Z = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    f = _gpu_decompose(ctx, Z, 4, 4, 32, 0, 0)
    assert ctx.poll_device_status() == 0
    for t in (f.U, f.V, f.S):
        assert torch.isfinite(t).all()
    assert not f.S.any() and not f.U.any()
    N = torch.ones(256, 256, dtype=torch.bfloat16, device="cuda")
    N[3, 5] = float("nan")
    _gpu_decompose(ctx, N, 4, 4, 256, 0, 0)
    assert ctx.poll_device_status() & metis_lib.DEV_NONFINITE


def test_decompose_validation(ctx, metis_lib):
    M = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    f = ctx.new_factors(256, 256, 4)
    with pytest.raises(metis_lib.MetisError):
        ctx.decompose(M, k=4, s=200, l_k=32, seed=0, operand_id=0, refresh=True, step=0, factors=f)
    with pytest.raises(metis_lib.MetisError):
        ctx.decompose(M, k=4, s=4, l_k=4, seed=0, operand_id=0, refresh=True, step=0, factors=f)


# ---- edge cases of the decomposition (each against the oracle)

def test_rank_one(ctx, metis_lib):
    """k = 1: one direction, the top singular pair of the sampled sketch."""
    cfg = synth.scaled_config("gpt2_small_mlp_up", l=1024, m=768, n=768)
    _compare(ctx, cfg, "X", 1, 8, 82, 0, 1)


def test_sketch_as_wide_as_the_sample(ctx, metis_lib):
    """k + s = l_k: the sketch Y is square (20 x 20) before CholQR."""
    cfg = synth.scaled_config("gpt2_small_mlp_up", l=1024, m=768, n=768)
    _compare(ctx, cfg, "X", 12, 8, 20, 0, 1)


def test_smallest_operand(ctx, metis_lib):
    """A 128 x 128 operand, sampled (l_k = 32) and unsampled (l_k = 128)."""
    cfg = synth.scaled_config("tiny_fwd", l=128, m=128, n=128)
    _compare(ctx, cfg, "X", 4, 4, 32, 0, 0)
    _compare(ctx, cfg, "X", 4, 4, 128, 0, 0)


def _duplicated_columns(rank, rows=256, cols=128, seed=3):
    """A bf16 matrix whose columns repeat `rank` random base columns (exact rank `rank`)."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((rows, rank)) * np.geomspace(50.0, 1.0, rank)
    pick = rng.integers(0, rank, size=cols)
    pick[:rank] = np.arange(rank)
    return torch.from_numpy(np.ascontiguousarray(base[:, pick])).to(torch.bfloat16).contiguous()


@pytest.mark.parametrize("k", [4, 6])
def test_rank_deficient_sketch_drops_directions(ctx, metis_lib, k):
    """Duplicated columns give M exact rank 5, so the sketch of width k + 4 (8 or 10) is
    rank-deficient: reading R9's drop rule runs on the device (CholQR pivots and
    eigenvalues at or below 1e-12 of the largest count as zero).  The recovered directions
    match the oracle's; with k = 6 > rank the sixth singular value is exactly 0 and its
    left factor column is zero, as in the oracle, and no numeric failure is raised."""
    Mt = _duplicated_columns(5)
    M = Mt.double().numpy()
    rows, cols = M.shape
    f = _gpu_decompose(ctx, Mt.cuda(), k, 4, 32, 1, 0)
    assert ctx.poll_device_status() == 0
    ref = decompose.refresh_basis(M, k, 4, 32, 1, 0, 0)
    U, S, V = decompose.step_factors(M, ref["V"])
    Y = M[ref["rows"]] @ ref["omega"].astype(np.float64)
    _, _, dropped = linalg.cholqr(Y)
    assert int(np.sum(dropped)) == k + 4 - 5   # the oracle drops the dependent sketch columns
    gV, gU, gS = f.V.cpu().double().numpy(), f.U.cpu().double().numpy(), f.S.cpu().double().numpy()[:k]
    r = min(k, 5)
    assert linalg.principal_cosines(gV[:, :r], V[:, :r]).min() >= COS
    assert linalg.principal_cosines(gU[:, :r], U[:, :r]).min() >= COS
    assert np.max(np.abs(gS[:r] - S[:r]) / S[0]) < 1e-3
    if k > 5:
        assert np.all(S[5:] == 0.0) and np.all(gS[5:] == 0.0)
        assert np.all(U[:, 5:] == 0.0) and np.all(gU[:, 5:] == 0.0)
    low = (gU * gS) @ gV.T
    if k >= 5:                                # rank 5 is captured whole
        assert np.linalg.norm(low - M) / np.linalg.norm(M) < 1e-3


def test_rank_deficient_step_gram_converges(ctx, metis_lib):
    """M of exact rank 20 and a per-step basis of k = 32: the Gram of P = M V has 12
    eigenvalues at rounding level, whose mutual entries the eigensolver leaves alone once
    they fall below 1e-13 of the largest diagonal entry (without that floor they rotate
    among themselves until the sweep limit).  No numeric failure; the 20 captured singular
    values and directions match the oracle's."""
    Mt = _duplicated_columns(20, rows=512, cols=256, seed=5)
    M = Mt.double().numpy()
    f = _gpu_decompose(ctx, Mt.cuda(), 32, 8, 512, 3, 0)           # refresh (unsampled sketch)
    assert ctx.poll_device_status() == 0
    V0 = f.V.cpu().double().numpy()
    _gpu_decompose(ctx, Mt.cuda(), 32, 8, 512, 3, 0, refresh=False, step=1, factors=f)
    assert ctx.poll_device_status() == 0
    U, S, V = decompose.step_factors(M, V0)
    gS = f.S.cpu().double().numpy()[:32]
    assert np.max(np.abs(gS[:20] - S[:20]) / S[0]) < 1e-3
    assert np.all(gS[20:] <= 1e-3 * gS[0])
    gV, gU = f.V.cpu().double().numpy(), f.U.cpu().double().numpy()
    assert linalg.principal_cosines(gV[:, :20], V[:, :20]).min() >= COS
    assert linalg.principal_cosines(gU[:, :20], U[:, :20]).min() >= COS
