"""The context's SM-count target (metis_set_sm_count_target).

A smaller target makes the persistent kernels launch fewer CTAs (each then takes more
tiles) and sizes the split-K counts for fewer SMs.  Contract:

* the fused GeMM and the residual quantizer give bit-identical outputs at any target
  (every output tile or block is formed by one CTA in the same order);
* the decomposition's singular values agree with the full-target ones to within the
  reordering of fp32 / fp64 split sums;
* targets outside {0} U [2, device SMs] are refused with METIS_ERR_ARG and leave the
  context usable; 0 restores the device's count.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4
from tests.gpu_helpers import load_nvfp4
from workloads import synth

pytestmark = pytest.mark.gpu


@pytest.fixture
def tctx(ctx):
    """The shared context, put back on the device's SM count whatever the test did."""
    yield ctx
    ctx.set_sm_count_target(0)


def _operand(ctx, outer, inner, rng):
    M = (rng.standard_normal((outer, inner)) * np.exp(rng.uniform(-1, 1, (outer, 1)))).astype(np.float32)
    codes, scales = nvfp4.quantize_blocks(M, 1.0)
    t = ctx.new_nvfp4(outer, inner)
    load_nvfp4(t, codes, scales, 1.0)
    return t


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_fused_gemm_identical_at_a_smaller_target(tctx, metis_lib, out):
    rng = np.random.default_rng(11)
    p, q, K, fold_k = 768, 1024, 1024, 128      # 12 pair tiles
    A, B = _operand(tctx, p, K, rng), _operand(tctx, q, K, rng)
    Fa = torch.randn(p, fold_k, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    Fb = torch.randn(q, fold_k, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()
    outs = []
    for target in (0, 4, 6, 0):                  # 2 and 3 CTA pairs, then the device's count again
        tctx.set_sm_count_target(target)
        C = torch.full((p, q), float("nan"), dtype=out, device="cuda")
        tctx.gemm_nvfp4(A, B, q, C, Fa, Fb, None)
        torch.cuda.synchronize()
        assert tctx.poll_device_status() == 0
        outs.append(C)
    tctx.set_sm_count_target(0)
    for C in outs[1:]:
        assert torch.equal(C, outs[0])


@pytest.mark.parametrize("rounding", [0, 1])
def test_quantizer_identical_at_a_smaller_target(tctx, metis_lib, rounding):
    cfg = synth.scaled_config("llama3_8b_mlp_up", l=1024, m=1024, n=1024)
    M = synth.operand_matrix(cfg, "X").cuda()
    rows, cols = M.shape
    f = tctx.new_factors(rows, cols, 64)
    tctx.decompose(M, k=64, s=8, l_k=82, seed=1, operand_id=0, refresh=True, step=0, factors=f)
    res = []
    for target in (0, 8):
        tctx.set_sm_count_target(target)
        row, col = tctx.new_nvfp4(rows, cols), tctx.new_nvfp4(cols, rows)
        tctx.residual_quantize_nvfp4(M, f, row, col, rounding=rounding, seed=3, operand_id=0, step=2)
        torch.cuda.synchronize()
        assert tctx.poll_device_status() == 0
        res.append((row, col))
    tctx.set_sm_count_target(0)
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a.codes, b.codes)
        assert torch.equal(a.scales, b.scales)
        assert torch.equal(a.tensor_scale, b.tensor_scale)


def test_decomposition_agrees_at_a_smaller_target(tctx, metis_lib):
    cfg = synth.scaled_config("llama3_8b_mlp_up", l=1024, m=1024, n=1024)
    M = synth.operand_matrix(cfg, "X").cuda()
    rows, cols = M.shape
    S = []
    for target in (0, 10):
        tctx.set_sm_count_target(target)
        f = tctx.new_factors(rows, cols, 64, 8, 82)
        tctx.decompose(M, k=64, s=8, l_k=82, seed=1, operand_id=0, refresh=True, step=0, factors=f)
        tctx.decompose(M, k=64, s=8, l_k=82, seed=1, operand_id=0, refresh=False, step=1, factors=f)
        torch.cuda.synchronize()
        assert tctx.poll_device_status() == 0
        S.append(f.S[:64].double().cpu().numpy())
    tctx.set_sm_count_target(0)
    assert np.max(np.abs(S[1] - S[0]) / S[0][0]) < 1e-5


def test_out_of_range_targets_are_refused(tctx, metis_lib):
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    for bad in (-1, 1, n_sm + 1):
        with pytest.raises(metis_lib.MetisError) as e:
            tctx.set_sm_count_target(bad)
        assert metis_lib.STATUS_NAMES[e.value.status] == "ERR_ARG"
    tctx.set_sm_count_target(n_sm)
    tctx.set_sm_count_target(0)
    rng = np.random.default_rng(3)
    A, B = _operand(tctx, 256, 256, rng), _operand(tctx, 256, 256, rng)
    C = torch.empty(256, 256, dtype=torch.float32, device="cuda")
    tctx.gemm_nvfp4(A, B, 256, C)
    torch.cuda.synchronize()
    assert tctx.poll_device_status() == 0
