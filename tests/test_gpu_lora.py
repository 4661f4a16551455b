"""LoRA-SVD linear projection on the GPU vs the oracle.

Parity contract:
* the NVFP4 codes of X, W_res and D (round to nearest, tensor scale chosen from the
  data) equal the oracle's bit for bit, so the products are compared against the
  oracle evaluated on its own quantization;
* T = M bf16(L) within relative Frobenius error 1e-5 (fp32 sums of exact bf16
  products against fp64);
* the fused product (FP4 GeMM + branch in the bf16 hi/lo fold, fp32 out) within 1e-4
  (fp32 accumulation over K plus the ~2^-17 relative hi/lo split of T); with beta = 0 it
  equals the fold-free FP4 GeMM bit for bit;
* branch gradients within 2e-5 (T as a bf16 hi/lo pair, fp32 sums);
* the constraint within 1e-5 (fp64 CholQR on both sides, fp32 outputs);
* the realignment: the branch singular values within 1e-3 of the oracle's (the
  decomposition's own contract), L2 orthonormal, and W_res + beta L2 L1 equal to the
  input's W_eff within fp32 rounding.
"""

import numpy as np
import pytest
import torch

from oracle import lora_svd, nvfp4
from tests.gpu_helpers import codes_unpacked, rel_fro
from workloads import synth

pytestmark = pytest.mark.gpu


def _bf16_matrix(rows, cols, rng, scale=1.0):
    return synth.to_bf16(synth.anisotropic(rows, cols, synth.n_spikes(rows, cols), 20.0, 0.9, rng) * scale)


def _quantize_both(ctx, M, op):
    row, col = ctx.new_nvfp4(*M.shape), ctx.new_nvfp4(M.shape[1], M.shape[0])
    ctx.residual_quantize_nvfp4(M, None, rowwise=row, colwise=col, rounding=0, operand_id=op, tensor_scale=0.0)
    return row, col


def _oracle_hat(M, orientation, gpu_t):
    """The oracle's own quantization of M (checked bit-exact against the GPU's) decoded."""
    M = np.asarray(M, dtype=np.float32)
    g = nvfp4.auto_tensor_scale(M)
    codes, scales = nvfp4.quantize_oriented(M, orientation, g=g, rounding="rn")
    gc, gs, gg = codes_unpacked(gpu_t)
    assert gg == g and np.array_equal(gc, codes) and np.array_equal(gs, scales)
    return nvfp4.dequantize_blocks(codes, scales, g)


@pytest.mark.parametrize("l,m,n,k", [(384, 512, 768, 16), (512, 768, 512, 64), (256, 256, 512, 5)])
def test_lora_linear_matches_oracle(ctx, l, m, n, k):
    rng = np.random.default_rng(l + m + n + k)
    X, W, D = _bf16_matrix(l, m, rng), _bf16_matrix(m, n, rng, 0.05), _bf16_matrix(l, n, rng, 1e-3)
    L2 = torch.from_numpy((rng.standard_normal((m, k)) / np.sqrt(m)).astype(np.float32))
    L1 = torch.from_numpy((rng.standard_normal((k, n)) * 0.1).astype(np.float32))
    beta = 0.75
    Xg, Wg, Dg, L2g, L1g = (t.cuda() for t in (X, W, D, L2, L1))
    xr, _ = _quantize_both(ctx, Xg, 0)
    wr, wc = _quantize_both(ctx, Wg, 1)
    dr, _ = _quantize_both(ctx, Dg, 2)
    Y = torch.empty(l, n, dtype=torch.float32, device="cuda")
    dX = torch.empty(l, m, dtype=torch.float32, device="cuda")
    Tx = torch.empty(l, k, dtype=torch.float32, device="cuda")
    Td = torch.empty(l, k, dtype=torch.float32, device="cuda")
    ctx.lora_linear(0, xr, wc, Xg, L2g, L1g, beta, Y, T=Tx)
    ctx.lora_linear(1, dr, wr, Dg, L2g, L1g, beta, dX, T=Td)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0

    Xn, Wn, Dn = X.double().numpy(), W.double().numpy(), D.double().numpy()
    x_hat = _oracle_hat(Xn, "row", xr)
    w_hat_col = _oracle_hat(Wn, "col", wc)      # n x m: Q(W)^T, K-major for the forward
    w_hat_row = _oracle_hat(Wn, "row", wr)      # m x n
    d_hat = _oracle_hat(Dn, "row", dr)
    Y_ref, Tx_ref = lora_svd.lora_linear(0, x_hat, w_hat_col, Xn, L2.numpy(), L1.numpy(), beta)
    dX_ref, Td_ref = lora_svd.lora_linear(1, d_hat, w_hat_row, Dn, L2.numpy(), L1.numpy(), beta)
    assert rel_fro(Tx.cpu().numpy(), Tx_ref) < 1e-5
    assert rel_fro(Td.cpu().numpy(), Td_ref) < 1e-5
    assert rel_fro(Y.cpu().numpy(), Y_ref) < 1e-4
    assert rel_fro(dX.cpu().numpy(), dX_ref) < 1e-4
    # the branch is a visible share of the product (the test would see a dropped term)
    assert rel_fro(Y_ref, x_hat @ w_hat_col.T) > 1e-2

    # bf16 output of the same product
    Yb = torch.empty(l, n, dtype=torch.bfloat16, device="cuda")
    ctx.lora_linear(0, xr, wc, Xg, L2g, L1g, beta, Yb)
    assert rel_fro(Yb.float().cpu().numpy(), Y_ref) < 5e-3

    # beta = 0: exactly the fold-free FP4 GeMM
    Y0 = torch.empty(l, n, dtype=torch.float32, device="cuda")
    Yp = torch.empty(l, n, dtype=torch.float32, device="cuda")
    ctx.lora_linear(0, xr, wc, Xg, L2g, L1g, 0.0, Y0)
    ctx.gemm_nvfp4(xr, wc, n, Yp)
    torch.cuda.synchronize()
    assert torch.equal(Y0, Yp)


@pytest.mark.parametrize("p,c,k", [(384, 512, 16), (256, 768, 64), (512, 256, 3)])
def test_branch_grad_matches_oracle(ctx, p, c, k):
    rng = np.random.default_rng(p * 7 + c + k)
    M = _bf16_matrix(p, c, rng)
    T = torch.from_numpy(rng.standard_normal((p, k)).astype(np.float32))
    beta = -1.5
    G = torch.empty(c, k, dtype=torch.float32, device="cuda")
    Gt = torch.empty(k, c, dtype=torch.float32, device="cuda")
    ctx.lora_branch_grad(M.cuda(), T.cuda(), beta, G)
    ctx.lora_branch_grad(M.cuda(), T.cuda(), beta, Gt, transpose_out=True)
    torch.cuda.synchronize()
    ref = lora_svd.branch_grad(M.double().numpy(), T.numpy(), beta)
    assert rel_fro(G.cpu().numpy(), ref) < 2e-5
    assert rel_fro(Gt.cpu().numpy(), ref.T) < 2e-5


@pytest.mark.parametrize("m,n,k", [(512, 768, 16), (256, 512, 64)])
def test_constraint_matches_oracle(ctx, m, n, k):
    rng = np.random.default_rng(m + n + k)
    L2 = (rng.standard_normal((m, k)) * np.linspace(0.1, 3.0, k)[None, :]).astype(np.float32)
    L1 = rng.standard_normal((k, n)).astype(np.float32)
    L2g, L1g = torch.from_numpy(L2).cuda(), torch.from_numpy(L1).cuda()
    ctx.lora_constrain(L2g, L1g)
    torch.cuda.synchronize()
    Q, L1n = lora_svd.constrain(L2, L1)
    assert rel_fro(L2g.cpu().numpy(), Q) < 1e-5
    assert rel_fro(L1g.cpu().numpy(), L1n) < 1e-5
    Qg = L2g.double().cpu().numpy()
    assert np.allclose(Qg.T @ Qg, np.eye(k), atol=1e-5)
    assert rel_fro(Qg @ L1g.double().cpu().numpy(), L2.astype(np.float64) @ L1) < 1e-5


def test_realign_matches_oracle(ctx, metis_lib):
    rng = np.random.default_rng(11)
    m, n, k, s, beta = 512, 768, 8, 8, 0.5
    U0, _ = np.linalg.qr(rng.standard_normal((m, k)))
    V0, _ = np.linalg.qr(rng.standard_normal((n, k)))
    S0 = 30.0 * 0.7 ** np.arange(k)
    W_res = (0.01 * rng.standard_normal((m, n))).astype(np.float32)
    L2 = (U0 * S0[None, :]).astype(np.float32)
    L1 = (V0.T / beta).astype(np.float32)
    Wg, L2g, L1g = (torch.from_numpy(a.copy()).cuda() for a in (W_res, L2, L1))
    f = metis_lib.Factors(m, n, k)
    Wb = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ctx.lora_realign(Wg, L2g, L1g, beta, f, Wb, s=s, l_k=m, seed=3, operand_id=1, step=0)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    W_eff = W_res.astype(np.float64) + beta * (L2.astype(np.float64) @ L1)
    Wn_ref, L2_ref, L1_ref, S_ref = lora_svd.realign(W_res, L2, L1, beta, k, s, seed=3, operand_id=1, step=0)
    gW, gL2, gL1 = (t.double().cpu().numpy() for t in (Wg, L2g, L1g))
    gS = f.S.double().cpu().numpy()[:k]
    assert np.max(np.abs(gS - S_ref) / S_ref[0]) < 1e-3
    assert np.allclose(gL2.T @ gL2, np.eye(k), atol=1e-4)
    assert rel_fro(gW + beta * gL2 @ gL1, W_eff) < 1e-6
    # the branch spans the oracle's (sign-fixed factors: column by column)
    assert rel_fro(gL2, L2_ref) < 1e-3
    assert rel_fro(gL1, L1_ref) < 1e-3
    assert rel_fro(gW, Wn_ref) < 1e-3 * np.linalg.norm(W_eff) / np.linalg.norm(Wn_ref)


def test_lora_svd_layer_trains(ctx):
    """A LoRASVDLinear regressing a fixed random linear teacher: the loss falls, the
    branch keeps orthonormal columns after every step, and the weight it represents
    is unchanged by the constraint and the realignment."""
    from spectral_quantized_gemm_b200.lora_svd import LoRASVDLinear
    torch.manual_seed(0)
    m, n, tokens = 256, 512, 512
    layer = LoRASVDLinear(m, n, k=8, realign_every=5).cuda()
    teacher = torch.randn(m, n, device="cuda") / m ** 0.5
    opt = torch.optim.Adam(layer.parameters(), lr=2e-3)
    losses = []
    for step in range(12):
        x = torch.randn(tokens, m, device="cuda")
        y = layer(x).float()
        loss = ((y - x @ teacher) ** 2).mean()
        opt.zero_grad()
        loss.backward()
        assert layer.L2.grad is not None and layer.L1.grad is not None and layer.W_res.grad is not None
        opt.step()
        with torch.no_grad():
            W_before = layer.W_res + layer.beta * layer.L2 @ layer.L1
        layer.post_step()
        with torch.no_grad():
            W_after = layer.W_res + layer.beta * layer.L2 @ layer.L1
            assert (W_after - W_before).norm() <= 1e-5 * W_before.norm()
            G = layer.L2.t() @ layer.L2
            assert torch.allclose(G, torch.eye(8, device="cuda"), atol=1e-4)
        losses.append(loss.item())
    assert ctx.poll_device_status() == 0
    assert losses[-1] < 0.8 * losses[0]


def test_lora_llama_up_full_size_sampled(ctx):
    """LLaMA-3 8B MLP-up at full size (the benchmark's LoRA-SVD launches, k = 64):
    256 sampled rows of Y and dX against the oracle on the decoded operands, the branch
    gradients dL2 in full and dL1 on 256 sampled columns."""
    from tests.gpu_helpers import dequant
    cfg = synth.CONFIGS["llama3_8b_mlp_up"]
    l, m, n, k, beta = cfg["l"], cfg["m"], cfg["n"], 64, 1.0
    X, W, D = (synth.operand_matrix(cfg, name) for name in ("X", "W", "D"))
    rng = np.random.default_rng(21)
    L2 = torch.from_numpy((rng.standard_normal((m, k)) / np.sqrt(m)).astype(np.float32))
    L1 = torch.from_numpy((rng.standard_normal((k, n)) * 0.05).astype(np.float32))
    Xg, Wg, Dg, L2g, L1g = (t.cuda() for t in (X, W, D, L2, L1))
    xr, _ = _quantize_both(ctx, Xg, 0)
    wr, wc = _quantize_both(ctx, Wg, 1)
    dr, _ = _quantize_both(ctx, Dg, 2)
    Y = torch.empty(l, n, dtype=torch.float32, device="cuda")
    dX = torch.empty(l, m, dtype=torch.float32, device="cuda")
    Tx = torch.empty(l, k, dtype=torch.float32, device="cuda")
    Td = torch.empty(l, k, dtype=torch.float32, device="cuda")
    ctx.lora_linear(0, xr, wc, Xg, L2g, L1g, beta, Y, T=Tx)
    ctx.lora_linear(1, dr, wr, Dg, L2g, L1g, beta, dX, T=Td)
    dL2 = torch.empty(m, k, dtype=torch.float32, device="cuda")
    dL1 = torch.empty(k, n, dtype=torch.float32, device="cuda")
    ctx.lora_branch_grad(Xg, Td, beta, dL2)
    ctx.lora_branch_grad(Dg, Tx, beta, dL1, transpose_out=True)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0

    rows = np.sort(rng.choice(l, 256, replace=False))
    Xn, Dn = X.double().numpy(), D.double().numpy()
    L2n, L1n = L2.numpy(), L1.numpy()
    x_hat = dequant(xr)[rows]
    Y_ref, Tx_rows = lora_svd.lora_linear(0, x_hat, dequant(wc), Xn[rows], L2n, L1n, beta)
    assert rel_fro(Y[rows].double().cpu().numpy(), Y_ref) < 1e-4
    assert rel_fro(Tx[rows].double().cpu().numpy(), Tx_rows) < 1e-5
    d_hat = dequant(dr)[rows]
    dX_ref, Td_rows = lora_svd.lora_linear(1, d_hat, dequant(wr), Dn[rows], L2n, L1n, beta)
    assert rel_fro(dX[rows].double().cpu().numpy(), dX_ref) < 1e-4
    assert rel_fro(Td[rows].double().cpu().numpy(), Td_rows) < 1e-5
    # the gradients from the oracle's own T (all rows)
    Td_all = lora_svd.branch_input(1, Dn, L2n, L1n)
    assert rel_fro(dL2.double().cpu().numpy(), lora_svd.branch_grad(Xn, Td_all, beta)) < 2e-5
    cols = np.sort(rng.choice(n, 256, replace=False))
    Tx_all = lora_svd.branch_input(0, Xn, L2n, L1n)
    ref_dl1 = lora_svd.branch_grad(Dn[:, cols], Tx_all, beta).T
    assert rel_fro(dL1[:, cols].double().cpu().numpy(), ref_dl1) < 2e-5


def test_lora_validation(ctx, metis_lib):
    """Host-side checks of the LoRA-SVD calls return their status before any launch, and
    the context stays usable afterwards."""
    l, m, n, k = 256, 256, 512, 8
    X = torch.zeros(l, m, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(m, n, dtype=torch.bfloat16, device="cuda")
    xr, _ = _quantize_both(ctx, X, 0)
    _, wc = _quantize_both(ctx, W, 1)
    L2 = torch.zeros(m, k, device="cuda")
    L1 = torch.zeros(k, n, device="cuda")
    Y = torch.empty(l, n, device="cuda")

    def status(fn, *args, **kw):
        with pytest.raises(metis_lib.MetisError) as e:
            fn(*args, **kw)
        return e.value.status

    assert status(ctx.lora_linear, 2, xr, wc, X, L2, L1, 1.0, Y) == 1                     # which
    assert status(ctx.lora_linear, 0, xr, wc, X, torch.zeros(m, 65, device="cuda"),
                  torch.zeros(65, n, device="cuda"), 1.0, Y) == 2                         # rank 65
    assert status(ctx.lora_linear, 0, xr, wc, X, L2, L1, float("nan"), Y) == 1           # beta
    w128c = ctx.new_nvfp4(128, m)     # a B operand with 128 output columns (never read)
    assert status(ctx.lora_linear, 0, xr, w128c, X, L2, torch.zeros(k, 128, device="cuda"), 1.0,
                  torch.empty(l, 128, device="cuda")) == 2                                # 128 output columns
    assert status(ctx.lora_linear, 0, xr, wc, X[:, :128], L2, L1, 1.0, Y) == 2           # M is not l x m
    assert status(ctx.lora_linear, 0, xr, wc, X, L2, L1, 1.0, torch.empty(l, n - 4, device="cuda")) == 3
    assert status(ctx.lora_branch_grad, torch.zeros(200, m, dtype=torch.bfloat16, device="cuda"),
                  torch.zeros(200, k, device="cuda"), 1.0, torch.zeros(m, k, device="cuda")) == 2
    assert status(ctx.lora_constrain, torch.zeros(200, k, device="cuda"), L1) == 2
    f = metis_lib.Factors(m, n, k)
    Wb = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    assert status(ctx.lora_realign, torch.zeros(m, n, device="cuda"), L2, L1, 0.0, f, Wb, s=8, l_k=m,
                  seed=0, operand_id=1, step=0) == 1                                      # beta = 0
    ctx.lora_linear(0, xr, wc, X, L2, L1, 1.0, Y)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0 and torch.count_nonzero(Y).item() == 0
