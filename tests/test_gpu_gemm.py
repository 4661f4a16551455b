"""Fused NVFP4 GeMM (+ bf16 rank-fold) vs the oracle on identical operands.

The oracle multiplies the dequantized operands in fp64 (FP4 x FP4 products are
exact); the GPU accumulates in fp32 in tensor memory.  Contract: relative
Frobenius error <= 2e-3 (the parity contract); the expected error is fp32 accumulation
only, so a much tighter internal bound (1e-4) is checked as well.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4
from tests.gpu_helpers import bf16_round, load_nvfp4, rel_fro

pytestmark = pytest.mark.gpu
TOL = 2e-3
TIGHT = 1e-4


def _operand(ctx, outer, inner, rng, g=1.0, valid_rows=None):
    M = (rng.standard_normal((outer, inner)) * np.exp(rng.uniform(-1, 1, (outer, 1)))).astype(np.float32)
    if valid_rows is not None:
        M[valid_rows:] = 0.0
    codes, scales = nvfp4.quantize_blocks(M, g)
    t = ctx.new_nvfp4(outer, inner)
    load_nvfp4(t, codes, scales, g)
    return t, nvfp4.dequantize_blocks(codes, scales, g)


def _run(ctx, p, q, K, fold_k=0, ga=1.0, gb=1.0, thin=False, col_scale=False, out=torch.float32, seed=0,
         with_abs=False):
    rng = np.random.default_rng(seed)
    A, Ad = _operand(ctx, p, K, rng, ga)
    B, Bd = _operand(ctx, 128 if thin else q, K, rng, gb, valid_rows=q if thin else None)
    want = Ad @ Bd[:q].T
    absprod = np.abs(Ad) @ np.abs(Bd[:q]).T
    Fa = Fb = None
    if fold_k:
        fa = torch.randn(p, fold_k, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
        fb = torch.randn(128 if thin else q, fold_k, generator=torch.Generator().manual_seed(seed + 1)).to(torch.bfloat16)
        fan, fbn = fa.double().numpy(), fb.double().numpy()[:q]
        want = want + ga * gb * (fan @ fbn.T)
        absprod = absprod + ga * gb * (np.abs(fan) @ np.abs(fbn).T)
        Fa, Fb = fa.cuda(), fb.cuda()
    cs = None
    if col_scale:
        csv = rng.uniform(0.5, 2.0, q).astype(np.float32)
        want = want * csv[None, :]
        absprod = absprod * csv[None, :]
        cs = torch.from_numpy(csv).cuda()
    C = torch.full((p, q), float("nan"), dtype=out, device="cuda")
    ctx.gemm_nvfp4(A, B, q, C, Fa, Fb, cs)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    if with_abs:
        return C.double().cpu().numpy(), want, absprod, K + fold_k
    return C.double().cpu().numpy(), want


@pytest.mark.parametrize("p,q,K", [(128, 256, 256), (256, 512, 768), (384, 768, 4096)])
def test_fp4_gemm(ctx, metis_lib, p, q, K):
    got, want = _run(ctx, p, q, K)
    err = rel_fro(got, want)
    assert err <= TOL and err <= TIGHT, err


def test_fp4_gemm_many_tiles_per_cta(ctx, metis_lib):
    """More output tiles than SMs: each persistent CTA runs several tiles."""
    got, want = _run(ctx, 2048, 4096, 512, seed=3)
    assert rel_fro(got, want) <= TIGHT


def test_pair_tiles_fold_column_scale_bf16(ctx, metis_lib):
    # CTA-pair path (both output dimensions multiples of 256): 4 x 9 pair tiles, a K loop
    # that wraps the stage ring, three fold stages, per-column scale, bf16 output
    got, want, absprod, terms = _run(ctx, 1024, 2304, 1536, fold_k=192, col_scale=True, out=torch.bfloat16,
                                     seed=21, with_abs=True)
    assert np.all(np.isfinite(got))
    # bf16 rounding of each output plus fp32 accumulation
    bound = np.abs(want) * 2.0 ** -8 + absprod * terms * 2.0 ** -23
    assert np.all(np.abs(got - want) <= bound)


@pytest.mark.parametrize("q", [16, 32, 64])
def test_thin_gemm_with_column_scale(ctx, metis_lib, q):
    got, want = _run(ctx, 512, q, 1024, thin=True, col_scale=True, seed=q)
    assert rel_fro(got, want) <= TIGHT


@pytest.mark.parametrize("fold_k", [64, 128, 256])
def test_fold_into_same_accumulator(ctx, metis_lib, fold_k):
    got, want = _run(ctx, 256, 512, 512, fold_k=fold_k, seed=fold_k)
    assert rel_fro(got, want) <= TIGHT


def test_fold_thin_and_tensor_scales(ctx, metis_lib):
    got, want = _run(ctx, 256, 64, 768, fold_k=64, ga=0.5, gb=4.0, thin=True, col_scale=True, seed=9)
    assert rel_fro(got, want) <= TIGHT
    got, want = _run(ctx, 256, 256, 256, fold_k=128, ga=2.0 ** -6, gb=0.25, seed=10)
    assert rel_fro(got, want) <= TIGHT


def test_bf16_output_is_the_rounded_result(ctx, metis_lib):
    """Each bf16 output is the fp32 accumulator rounded once: within half a bf16 ulp
    (2^-9 relative) plus the worst-case fp32 accumulation error of its dot product."""
    got, want, absprod, terms = _run(ctx, 256, 512, 1024, fold_k=64, out=torch.bfloat16, seed=4, with_abs=True)
    bound = 2.0 ** -8 * np.abs(want) + terms * 2.0 ** -24 * absprod * 1.01
    assert np.all(np.abs(got - want) <= bound)
    assert np.mean(got == bf16_round(want)) > 0.99


def test_gemm_validation(ctx, metis_lib):
    rng = np.random.default_rng(0)
    A, _ = _operand(ctx, 128, 256, rng)
    B, _ = _operand(ctx, 256, 512, rng)
    C = torch.zeros(128, 256, device="cuda")
    with pytest.raises(metis_lib.MetisError):
        ctx.gemm_nvfp4(A, B, 256, C)          # K mismatch
    B2, _ = _operand(ctx, 200 - 72, 256, rng)
    with pytest.raises(metis_lib.MetisError):
        ctx.gemm_nvfp4(A, B2, 48, C)          # thin width not in {16, 32, 64}


def test_mma_peak_microbenchmark(ctx, metis_lib):
    """The no-memory-traffic NVFP4 MMA loop runs cleanly and reports a rate between the
    fused GeMM's and the nominal dense FP4 peak (about 9.5 PFLOP/s at 1.965 GHz)."""
    rate = ctx.nvfp4_mma_peak(iters=1024, reps=3)
    assert ctx.poll_device_status() == 0
    assert 2000.0 < rate < 12000.0, rate
    with pytest.raises(metis_lib.MetisError):
        ctx.nvfp4_mma_peak(iters=0)
