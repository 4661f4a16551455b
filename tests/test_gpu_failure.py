"""Failure detection, output bounds and checkpoint/resume on the GPU.

* A bounded wait that runs out is reported as METIS_DEV_TIMEOUT and leaves the context
  usable (the self-test waits on a barrier nothing arrives at; nothing faults or hangs).
* An eigensolve that stops unconverged is reported as METIS_DEV_NUMERIC (the self-test
  allows it no sweep) and leaves the context usable.
* NaN canaries around output buffers: the fused GeMM (CTA-pair and single-CTA paths, bf16
  and fp32) and the residual quantizer write every element they own and nothing beyond.
* MetisLinear resumed from a checkpoint after 4 steps gives the same step-8 results, bit
  for bit, as 8 uninterrupted steps.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4
from tests.gpu_helpers import codes_unpacked

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_survives(ctx, metis_lib):
    assert ctx.poll_device_status() == 0
    ctx.selftest_wait_timeout(1_000_000)
    st = ctx.poll_device_status()
    assert st & metis_lib.DEV_TIMEOUT
    assert ctx.poll_device_status() == 0          # cleared by the read
    # the context still works: plain NVFP4 of a small matrix is bit-exact with the oracle
    rng = np.random.default_rng(1)
    R = rng.standard_normal((128, 256)).astype(np.float32)
    t = ctx.new_nvfp4(128, 256)
    ctx.quantize_nvfp4_f32(torch.from_numpy(R).cuda(), t, None)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    codes, scales, _ = codes_unpacked(t)
    wc, ws = nvfp4.quantize_oriented(R, "row")
    assert np.array_equal(codes, wc) and np.array_equal(scales, ws)
    with pytest.raises(metis_lib.MetisError):
        ctx.selftest_wait_timeout(0)


def test_numeric_failure_is_reported_and_the_context_survives(ctx, metis_lib):
    """An eigensolve that reaches its sweep limit unconverged latches METIS_DEV_NUMERIC
    (the self-test allows it no sweep); the bit clears on read and a decomposition right
    after is clean and agrees with the oracle's singular values."""
    from oracle import decompose
    from workloads import synth
    assert ctx.poll_device_status() == 0
    ctx.selftest_numeric()
    st = ctx.poll_device_status()
    assert st & metis_lib.DEV_NUMERIC
    assert not st & (metis_lib.DEV_TIMEOUT | metis_lib.DEV_NONFINITE)
    assert ctx.poll_device_status() == 0          # cleared by the read
    cfg = synth.CONFIGS["tiny_fwd"]
    Mt = synth.operand_matrix(cfg, "X")
    f = ctx.new_factors(256, 256, 4, 4, 32)
    ctx.decompose(Mt.cuda(), k=4, s=4, l_k=32, seed=0, operand_id=0, refresh=True, step=0, factors=f)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    M = Mt.double().numpy()
    ref = decompose.refresh_basis(M, 4, 4, 32, 0, 0, 0)
    _, S, _ = decompose.step_factors(M, ref["V"])
    gS = f.S.cpu().double().numpy()[:4]
    assert np.max(np.abs(gS - S) / S[0]) < 1e-3


def _operand(ctx, outer, inner, seed):
    rng = np.random.default_rng(seed)
    M = torch.from_numpy(rng.standard_normal((outer, inner)).astype(np.float32)).to(torch.bfloat16).cuda()
    t = ctx.new_nvfp4(outer, inner)
    ctx.residual_quantize_nvfp4(M, None, rowwise=t)
    return t


@pytest.mark.parametrize("p,q,dtype", [(512, 768, torch.bfloat16), (512, 768, torch.float32),
                                       (384, 256, torch.bfloat16), (384, 256, torch.float32)])
def test_gemm_writes_exactly_its_output(ctx, metis_lib, p, q, dtype):
    """(512, 768) runs on CTA pairs, (384, 256) on single CTAs; C sits inside a wider
    NaN-filled buffer (ldc = q + 64) with a NaN row band below it."""
    K = 512
    A, B = _operand(ctx, p, K, 1), _operand(ctx, q, K, 2)
    big = torch.full((p + 8, q + 64), float("nan"), dtype=dtype, device="cuda")
    C = big[:p, :q]
    ctx.gemm_nvfp4(A, B, q, C)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    assert torch.isfinite(big[:p, :q]).all()
    assert torch.isnan(big[:p, q:]).all() and torch.isnan(big[p:]).all()


def test_quantizer_writes_exactly_its_output(ctx, metis_lib):
    rows, cols = 384, 512
    M = torch.randn(rows, cols, device="cuda").to(torch.bfloat16)
    f = ctx.new_factors(rows, cols, 16)
    ctx.decompose(M, k=16, s=8, l_k=64, seed=1, operand_id=0, refresh=True, step=0, factors=f)
    outs = []
    for outer, inner in ((rows, cols), (cols, rows)):
        nc, ns = outer * inner // 2, metis_lib.Nvfp4(outer, inner).scales.numel()
        codes = torch.full((nc + 512,), 0xA5, dtype=torch.uint8, device="cuda")
        scales = torch.full((ns + 512,), 0x5A, dtype=torch.uint8, device="cuda")
        g = torch.full((8,), float("nan"), device="cuda")
        t = metis_lib.Nvfp4(outer, inner)
        t.codes, t.scales, t.tensor_scale = codes[:nc], scales[:ns], g[:4]
        t.struct = metis_lib.Nvfp4Struct(codes.data_ptr(), scales.data_ptr(), g.data_ptr(), outer, inner)
        outs.append((t, codes, scales, g, nc, ns))
    ctx.residual_quantize_nvfp4(M, f, outs[0][0], outs[1][0], rounding=1, seed=3)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    for t, codes, scales, g, nc, ns in outs:
        assert (codes[nc:] == 0xA5).all() and (scales[ns:] == 0x5A).all()
        assert g[0].item() == 1.0 and torch.isnan(g[1:]).all()


def _run_steps(layer, steps, start=0):
    outs = []
    for t in range(start, start + steps):
        g = torch.Generator(device="cuda").manual_seed(100 + t)
        x = torch.randn(1024, 512, device="cuda", generator=g).to(torch.bfloat16).requires_grad_(True)
        dy = (torch.randn(1024, 768, device="cuda", generator=g) * 1e-3).to(torch.bfloat16)
        layer.weight.grad = None
        y = layer(x)
        y.backward(dy)
        outs.append((y.detach().clone(), x.grad.clone(), layer.weight.grad.clone()))
    return outs


def test_linear_resumes_bit_for_bit_from_a_checkpoint(ctx, metis_lib, tmp_path):
    from spectral_quantized_gemm_b200.linear import MetisLinear
    torch.manual_seed(0)
    a = MetisLinear(512, 768, k=16, refresh_every=3, seed=4, device="cuda")
    b = MetisLinear(512, 768, k=16, refresh_every=3, seed=4, device="cuda")
    b.load_state_dict(a.state_dict())
    straight = _run_steps(a, 8)
    _run_steps(b, 4)
    torch.save(b.state_dict(), tmp_path / "metis.pt")
    c = MetisLinear(512, 768, k=16, refresh_every=3, seed=4, device="cuda")
    c.load_state_dict(torch.load(tmp_path / "metis.pt", weights_only=False))
    assert c.step == 4
    resumed = _run_steps(c, 4, start=4)
    for (y0, dx0, dw0), (y1, dx1, dw1) in zip(straight[4:], resumed):
        assert torch.equal(y0, y1) and torch.equal(dx0, dx1) and torch.equal(dw0, dw1)
