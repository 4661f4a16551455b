"""MetisLinear, the torch.autograd wrapper over the C ABI, on the GPU.

1. Its Y, dX and dW are exactly the C-ABI call sequence it stands for: decomposition
   and residual quantization of X, W and dY with the layer's seed, operand ids and step,
   then metis_linear_fwd / metis_linear_bwd.
2. Between refreshes it reuses the basis of the previous step (training strategy of the
   method: decompose every few steps, reuse the basis in between).
3. A short training run of a GPT-2-small MLP block on synthetic tokens follows the bf16
   run of the same model, optimizer and data.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _tokens(rows, cols, seed):
    """Synthetic activations: N(0,1) bulk plus a few large outlier channels."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(rows, cols, device="cuda", generator=g)
    ch = torch.randperm(cols, generator=torch.Generator().manual_seed(seed))[: max(1, cols // 50)]
    x[:, ch.cuda()] *= 20.0
    return x


def _reference_operand(ctx, M, k, s, l_k, seed, op, step, refresh, V=None):
    rows, cols = M.shape
    f = ctx.new_factors(rows, cols, k)
    if V is not None:
        f.V.copy_(V)
    ctx.decompose(M, k=k, s=s, l_k=l_k, seed=seed, operand_id=op, refresh=refresh, step=step, factors=f,
                  rounding=1)
    row, col = ctx.new_nvfp4(rows, cols), ctx.new_nvfp4(cols, rows)
    ctx.residual_quantize_nvfp4(M, f, row, col, rounding=1, seed=seed, operand_id=op, step=step, tensor_scale=0.0)
    return f, row, col, ctx.operand(row, col, f)


def _reference_step(ctx, layer, x, dy, step, refresh, bases=None):
    """The C-ABI sequence of one MetisLinear step; returns Y, dX, dW and the new bases."""
    k, s = layer.k, layer.s
    w = layer.weight.detach().to(torch.bfloat16).contiguous()
    l, m = x.shape
    bases = bases or {}
    ops = {}
    for op, (name, M, l_k) in enumerate((("X", x, layer._l_k(l, True)), ("W", w, m),
                                         ("D", dy, layer._l_k(l, True)))):
        ops[name] = _reference_operand(ctx, M, k, s, l_k, layer.seed, op, step, refresh, bases.get(name))
    Y = torch.empty(l, layer.out_features, dtype=torch.bfloat16, device="cuda")
    ctx.linear_fwd(ops["X"][3], ops["W"][3], Y)
    dX = torch.empty(l, m, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(m, layer.out_features, dtype=torch.float32, device="cuda")
    ctx.linear_bwd(ops["X"][3], ops["W"][3], ops["D"][3], dX, dW)
    return Y, dX, dW, {n: o[0].V.clone() for n, o in ops.items()}


def test_wrapper_is_the_c_abi_sequence(ctx, metis_lib):
    from spectral_quantized_gemm_b200.linear import MetisLinear
    torch.manual_seed(0)
    layer = MetisLinear(768, 3072, seed=7, device="cuda")
    assert layer.k == 12
    bases = None
    for step in range(3):        # a refresh, then two steps that reuse the basis
        x = _tokens(2048, 768, 100 + step).to(torch.bfloat16).requires_grad_(True)
        dy = (_tokens(2048, 3072, 200 + step) * 1e-3).to(torch.bfloat16)
        layer.weight.grad = None
        y = layer(x)
        y.backward(dy)
        Y, dX, dW, bases = _reference_step(ctx, layer, x.detach(), dy, step, step == 0, bases)
        torch.cuda.synchronize()
        assert torch.equal(y, Y), f"step {step}: Y"
        assert torch.equal(x.grad, dX), f"step {step}: dX"
        assert layer.weight.grad.dtype == torch.float32
        assert torch.equal(layer.weight.grad, dW), f"step {step}: dW"
        assert ctx.poll_device_status() == 0
    assert layer.step == 3


def _oracle_operand(o):
    """The oracle's view of one of MetisLinear's own operands: its decoded residual codes
    and scales in both orientations, its quantized factors and singular values."""
    from tests.gpu_helpers import codes_unpacked
    k = o.factors.k
    cu, su, gu = codes_unpacked(o.factors.Uq)
    cv, sv, gv = codes_unpacked(o.factors.Vq)
    return {"row": codes_unpacked(o.row), "col": codes_unpacked(o.col), "U": True,
            "Uq": (cu[:k], su[:k], gu), "Vq": (cv[:k], sv[:k], gv), "S": o.factors.S.cpu().double().numpy()[:k]}


def test_wrapper_matches_the_oracle(ctx, metis_lib):
    """MetisLinear's Y, dX and dW against the oracle's product (oracle/metis.py) fed the
    layer's own codes, scales and factors, over a refresh and a reuse step: dW (fp32) within
    the 2e-3 contract, Y and dX (bf16) within it against the oracle rounded to bf16.  Every
    operand's decode tensor scale is the one reading R1b chooses from the data
    (oracle/nvfp4.py::auto_tensor_scale of the bf16 operand)."""
    from oracle import metis, nvfp4
    from tests.gpu_helpers import bf16_round, rel_fro
    from spectral_quantized_gemm_b200.linear import MetisLinear
    torch.manual_seed(1)
    layer = MetisLinear(768, 1024, k=12, seed=5, device="cuda")
    recorded = []
    prepare = layer._prepare

    def record(lib, M, op_id, step, sampled):
        o = prepare(lib, M, op_id, step, sampled)
        recorded.append((op_id, M.detach().clone(), o))
        return o

    layer._prepare = record
    for step in range(2):
        recorded.clear()
        x = _tokens(1024, 768, 300 + step).to(torch.bfloat16).requires_grad_(True)
        dy = (_tokens(1024, 1024, 400 + step) * 1e-4).to(torch.bfloat16)
        layer.weight.grad = None
        y = layer(x)
        y.backward(dy)
        torch.cuda.synchronize()
        assert ctx.poll_device_status() == 0
        ops = {op_id: (M, o) for op_id, M, o in recorded}
        assert sorted(ops) == [0, 1, 2]
        for op_id, (M, o) in ops.items():
            g = nvfp4.auto_tensor_scale(M.float().cpu().numpy())
            assert float(o.row.tensor_scale[0]) == g and float(o.col.tensor_scale[0]) == g, (step, op_id)
        ox, ow, od = (_oracle_operand(ops[i][1]) for i in range(3))
        Y = metis.linear_fwd(ox, ow)
        dX, dW = metis.linear_bwd(ox, ow, od)
        assert rel_fro(layer.weight.grad.double().cpu().numpy(), dW) <= 2e-3, step
        for got, want in ((y, Y), (x.grad, dX)):
            assert rel_fro(got.detach().double().cpu().numpy(), bf16_round(want)) <= 2e-3, step


def test_refresh_schedule_and_basis_reuse(ctx, metis_lib):
    from spectral_quantized_gemm_b200.linear import MetisLinear
    layer = MetisLinear(512, 768, k=16, refresh_every=2, seed=3, device="cuda")
    x0 = _tokens(1024, 512, 1).to(torch.bfloat16)
    V_prev = None
    for step in range(4):
        x = x0 + 0.1 * _tokens(1024, 512, 10 + step).to(torch.bfloat16)
        layer(x).backward((_tokens(1024, 768, 20 + step) * 1e-3).to(torch.bfloat16))
        V = layer._bases[0].V.clone().double()
        if V_prev is not None:
            if step % 2:
                # reuse step: V <- V V_r rotates the basis within the same subspace
                cos = torch.linalg.svdvals(V_prev.T @ V)
                assert cos.min() > 0.999, (step, cos.min().item())
            else:
                # refresh: a new sketch from other sampled rows (24 of 1024 here), so the
                # span moves; the 10 outlier channels' directions (the leading singular
                # directions of x0) are found again to the sampling's accuracy (the
                # method reports about 0.9 alignment at 1% sampling)
                cos = torch.linalg.svdvals(V_prev[:, :8].T @ V[:, :10])
                assert 0.75 < cos.min() < 0.999, (step, cos.min().item())
        V_prev = V
    assert layer.step == 4


def test_training_tracks_bf16(metis_lib):
    """GPT-2-small MLP block (768 -> 3072 -> GELU -> 768) regressing a fixed random
    teacher on synthetic tokens, 150 Adam steps, Metis W4A4G4 layers against bf16."""
    from spectral_quantized_gemm_b200.linear import MetisLinear
    torch.manual_seed(0)
    d, h, l, steps = 768, 3072, 4096, 150
    t1 = torch.randn(d, h, device="cuda") / d ** 0.5
    t2 = torch.randn(h, d, device="cuda") / h ** 0.5
    up, down = MetisLinear(d, h, seed=1, device="cuda"), MetisLinear(h, d, seed=2, device="cuda")
    w1 = torch.nn.Parameter(up.weight.detach().clone())
    w2 = torch.nn.Parameter(down.weight.detach().clone())
    opt_m = torch.optim.Adam(list(up.parameters()) + list(down.parameters()), lr=1e-3)
    opt_b = torch.optim.Adam([w1, w2], lr=1e-3)
    curves = {"metis": [], "bf16": []}
    for step in range(steps):
        x = _tokens(l, d, 1000 + step) * 0.2
        target = torch.nn.functional.gelu(x @ t1) @ t2
        xb = x.to(torch.bfloat16)
        ym = down(torch.nn.functional.gelu(up(xb)))
        loss_m = torch.nn.functional.mse_loss(ym.float(), target)
        opt_m.zero_grad()
        loss_m.backward()
        opt_m.step()
        yb = torch.nn.functional.gelu(xb @ w1.to(torch.bfloat16)) @ w2.to(torch.bfloat16)
        loss_b = torch.nn.functional.mse_loss(yb.float(), target)
        opt_b.zero_grad()
        loss_b.backward()
        opt_b.step()
        curves["metis"].append(loss_m.item())
        curves["bf16"].append(loss_b.item())
    m, b = np.array(curves["metis"]), np.array(curves["bf16"])
    print(f"loss start {m[0]:.4f} / {b[0]:.4f}; last 10 steps metis {m[-10:].mean():.5f}, bf16 {b[-10:].mean():.5f}")
    assert np.all(np.isfinite(m))
    assert m[-10:].mean() < 0.5 * m[:5].mean()          # it learns
    assert m[-10:].mean() < 1.25 * b[-10:].mean()       # and follows bf16
