"""GPU NVFP4 quantizer vs the oracle: codes and scales bit-exact on identical fp32 input.

Contract: NVFP4 codes and scales bit-exact given an identical fp32
residual input; both orientations; round-to-nearest and stochastic rounding.
"""

import numpy as np
import pytest
import torch

from oracle import formats, nvfp4
from tests.gpu_helpers import codes_unpacked

pytestmark = pytest.mark.gpu


def _inputs(rows, cols, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        return (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-3, 3, (rows, 1)))).astype(np.float32)
    if kind == "heavy":     # outlier columns, like anisotropic activations
        M = rng.standard_normal((rows, cols))
        M[:, rng.choice(cols, 4, replace=False)] *= 60
        return M.astype(np.float32)
    if kind == "ties":      # values on E2M1 midpoints and grid points of exact scales
        grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6])
        v = grid[rng.integers(0, len(grid), (rows, cols))] * rng.choice([-1.0, 1.0], (rows, cols))
        v[:, ::16] = 6.0
        v[::16, :] = 6.0
        return (v * 2.0 ** rng.integers(-4, 4, (rows, 1))).astype(np.float32)
    if kind == "edge":      # zeros, negative zeros, tiny and huge blocks
        M = rng.standard_normal((rows, cols)).astype(np.float32)
        M[0:4, :] = 0.0
        M[4, :] = -0.0
        M[5:9, :] *= 1e-7
        M[9:12, :] *= 1e4
        M[:, 0:16] = 0.0
        M[12, 16:32] = -0.0
        return M
    raise ValueError(kind)


def _check(ctx, metis_lib, R, rounding, g, seed=7, op=1, step=3):
    rows, cols = R.shape
    dev = torch.from_numpy(R).cuda()
    row = ctx.new_nvfp4(rows, cols)
    col = ctx.new_nvfp4(cols, rows)
    ctx.quantize_nvfp4_f32(dev, row, col, rounding=rounding, seed=seed, operand_id=op, step=step, tensor_scale=g)
    torch.cuda.synchronize()
    mode = "sr" if rounding else "rn"
    for t, orient in ((row, "row"), (col, "col")):
        codes, scales, gg = codes_unpacked(t)
        want_c, want_s = nvfp4.quantize_oriented(R, orient, g=g, rounding=mode, seed=seed, operand_id=op, step=step)
        assert gg == g
        assert np.array_equal(scales, want_s), (orient, mode)
        mism = np.argwhere(codes != want_c)
        assert len(mism) == 0, (orient, mode, mism[:5])


@pytest.mark.parametrize("kind", ["gauss", "heavy", "ties", "edge"])
@pytest.mark.parametrize("rounding", [0, 1])
def test_quantizer_bit_exact(ctx, metis_lib, kind, rounding):
    _check(ctx, metis_lib, _inputs(256, 384, kind, 11), rounding, 1.0)


@pytest.mark.parametrize("g", [0.25, 4.0])
def test_quantizer_tensor_scale(ctx, metis_lib, g):
    _check(ctx, metis_lib, _inputs(128, 256, "gauss", 3), 1, g)
    _check(ctx, metis_lib, _inputs(128, 256, "ties", 4), 0, g)


def test_quantizer_dense_cvt_sweep(ctx, metis_lib):
    """E2M1 decisions on a dense sweep of scaled values x in [-7, 7]: each row-wise
    block starts with 6.0, which pins its scale to 1, so x = v exactly."""
    rows = 512
    nblk = rows * 16
    M = np.empty((nblk, 16), np.float32)
    M[:, 0] = 6.0
    M[:, 1:] = np.linspace(-7.0, 7.0, nblk * 15).astype(np.float32).reshape(nblk, 15)
    M = np.ascontiguousarray(M.reshape(rows, 256))
    _check(ctx, metis_lib, M, 0, 1.0)
    _check(ctx, metis_lib, M, 1, 1.0)


def test_quantizer_full_size_sampled_rows(ctx, metis_lib):
    """LLaMA-3 8B gradient shape (8192 x 14336) in one launch; sampled rows and
    columns are recomputed by the oracle."""
    from oracle import philox
    rows, cols = 8192, 14336
    gen = torch.Generator(device="cuda").manual_seed(5)
    dev = torch.randn(rows, cols, device="cuda", generator=gen) * 3
    row = ctx.new_nvfp4(rows, cols)
    col = ctx.new_nvfp4(cols, rows)
    ctx.quantize_nvfp4_f32(dev, row, col, rounding=1, seed=2, operand_id=2, step=9)
    torch.cuda.synchronize()
    R = dev.cpu().numpy()
    codes = row.codes.view(rows, cols // 2)
    for i in np.random.default_rng(0).choice(rows, 24, replace=False):
        u = philox.sr_fields_at(2, 2, philox.SR_SUB_ROWWISE, 9, np.arange(i * cols, (i + 1) * cols))
        want_c, _ = nvfp4.quantize_blocks(R[i:i + 1], 1.0, "sr", u[None, :])
        assert np.array_equal(nvfp4.unpack_codes(codes[i:i + 1].cpu().numpy()), want_c)
    colcodes = col.codes.view(cols, rows // 2)
    for j in np.random.default_rng(1).choice(cols, 24, replace=False):
        u = philox.sr_fields_at(2, 2, philox.SR_SUB_COLWISE, 9, np.arange(j * rows, (j + 1) * rows))
        want_c, _ = nvfp4.quantize_blocks(np.ascontiguousarray(R[:, j][None, :]), 1.0, "sr", u[None, :])
        assert np.array_equal(nvfp4.unpack_codes(colcodes[j:j + 1].cpu().numpy()), want_c)


def test_nonfinite_input_sets_status(ctx, metis_lib):
    R = np.ones((128, 128), dtype=np.float32)
    R[5, 7] = np.nan
    row = ctx.new_nvfp4(128, 128)
    assert ctx.poll_device_status() == 0
    ctx.quantize_nvfp4_f32(torch.from_numpy(R).cuda(), row, None)
    assert ctx.poll_device_status() & metis_lib.DEV_NONFINITE
    assert ctx.poll_device_status() == 0


def test_host_validation(ctx, metis_lib):
    R = torch.zeros(128, 200, device="cuda")
    row = ctx.new_nvfp4(128, 200)
    with pytest.raises(metis_lib.MetisError) as e:
        ctx.quantize_nvfp4_f32(R, row, None)
    assert e.value.status == 2
    R = torch.zeros(128, 128, device="cuda")
    with pytest.raises(metis_lib.MetisError) as e:
        ctx.quantize_nvfp4_f32(R, ctx.new_nvfp4(128, 128), None, tensor_scale=0.3)
    assert e.value.status == 1
    with pytest.raises(metis_lib.MetisError):
        ctx.quantize_nvfp4_f32(R, ctx.new_nvfp4(256, 128), None)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7])
def test_dequantize_is_exact(ctx, metis_lib, g):
    """metis_dequantize_nvfp4 gives e2m1(code) * e4m3(scale) * g exactly (oracle decode)."""
    rng = np.random.default_rng(4)
    R = (rng.standard_normal((256, 512)) * np.exp(rng.uniform(-3, 3, (256, 1))) * g).astype(np.float32)
    t = ctx.new_nvfp4(256, 512)
    ctx.quantize_nvfp4_f32(torch.from_numpy(R).cuda(), t, None, rounding=1, seed=2, tensor_scale=g)
    out = ctx.dequantize_nvfp4(t)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    codes, scales, g_dev = codes_unpacked(t)
    assert g_dev == g
    want = nvfp4.dequantize_blocks(codes, scales, g_dev)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), want)
