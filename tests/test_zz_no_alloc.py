"""The allocation-free residual quantizer gives the same codes and scales as
the regular entry point.

Callers that may not allocate device memory while they run (CUDA graph capture,
frameworks that own device memory through their own allocator) use
metis_residual_quantize_nvfp4_noalloc, whose scratch is a fixed device array
inside the library.  This file is collected last on purpose.  Each check runs
the new entry point through the C ABI twice in a row, on different operands,
so a stale scratch from the previous call would show up.
"""

import pytest
import torch

from workloads import synth

pytestmark = pytest.mark.gpu


def _operand(ctx, cfg, name, k, seed):
    M = synth.operand_matrix(cfg, name).cuda()
    rows, cols = M.shape
    f = None
    if k:
        f = ctx.new_factors(rows, cols, k)
        l_k = cfg["l_k"] if name != "W" else rows
        ctx.decompose(M, k=k, s=cfg["s"], l_k=l_k, seed=seed, operand_id=0, refresh=True, step=0, factors=f)
    return M, f


def _both(ctx, M, f, noalloc, rounding, seed, tensor_scale=1.0):
    rows, cols = M.shape
    row, col = ctx.new_nvfp4(rows, cols), ctx.new_nvfp4(cols, rows)
    fn = ctx.residual_quantize_nvfp4_noalloc if noalloc else ctx.residual_quantize_nvfp4
    fn(M, f, row, col, rounding=rounding, seed=seed, operand_id=1, step=3, tensor_scale=tensor_scale)
    return row, col


def test_noalloc_matches_regular_entry(ctx, metis_lib):
    cfg = synth.scaled_config("gpt2_small_mlp_up", l=1024, m=768, n=768)
    cases = [_operand(ctx, cfg, "X", cfg["k"], 1), _operand(ctx, cfg, "W", 4, 2), _operand(ctx, cfg, "D", 0, 3)]
    for rounding in (1, 0):
        for M, f in cases:                       # calls in a row share the scratch
            a_row, a_col = _both(ctx, M, f, True, rounding, 7)
            b_row, b_col = _both(ctx, M, f, False, rounding, 7)
            torch.cuda.synchronize()
            assert ctx.poll_device_status() == 0
            for a, b in ((a_row, b_row), (a_col, b_col)):
                assert torch.equal(a.codes, b.codes)
                assert torch.equal(a.scales, b.scales)
                assert torch.equal(a.tensor_scale[:1], b.tensor_scale[:1])


def test_noalloc_rejects_shapes_beyond_its_scratch(ctx, metis_lib):
    M = torch.zeros(16384, 8320, dtype=torch.bfloat16, device="cuda")
    row, col = ctx.new_nvfp4(16384, 8320), ctx.new_nvfp4(8320, 16384)
    with pytest.raises(metis_lib.MetisError) as e:
        ctx.residual_quantize_nvfp4_noalloc(M, None, row, col)
    assert e.value.status == 2 and "24576" in str(e.value)


def test_noalloc_tensor_scale_chosen_from_the_data(ctx, metis_lib):
    """tensor_scale = 0 (g chosen from the data, its amax word kept in the fixed scratch):
    the same codes, scales and g as the regular entry point, g equal to the oracle's
    auto_tensor_scale, at k = 0 and k > 0, two calls in a row on differently scaled
    operands so a stale amax word would show."""
    from oracle import nvfp4
    cfg = synth.scaled_config("gpt2_small_mlp_up", l=1024, m=768, n=768)
    base = [_operand(ctx, cfg, "X", 0, 1), _operand(ctx, cfg, "W", cfg["k"], 2)]
    for scale in (2.0 ** -20, 2.0 ** 6):
        for M0, f in base:
            M = (M0.float() * scale).to(torch.bfloat16)      # powers of two keep the bf16 values exact
            if f is not None:
                ctx.decompose(M, k=f.k, s=cfg["s"], l_k=M.shape[0], seed=2, operand_id=0, refresh=True, step=0,
                              factors=f)
            a_row, a_col = _both(ctx, M, f, True, 1, 7, tensor_scale=0.0)
            b_row, b_col = _both(ctx, M, f, False, 1, 7, tensor_scale=0.0)
            torch.cuda.synchronize()
            assert ctx.poll_device_status() == 0
            g = nvfp4.auto_tensor_scale(M.float().cpu().numpy())
            for a, b in ((a_row, b_row), (a_col, b_col)):
                assert torch.equal(a.codes, b.codes)
                assert torch.equal(a.scales, b.scales)
                assert float(a.tensor_scale[0]) == g == float(b.tensor_scale[0])
