"""LoRA-SVD linear projection: W = W_res + beta L2 L1 (TEST INFRASTRUCTURE).

Source: "Full-Stack FP4: stable LLM pretraining with quantized projections,
optimizer and attention" (gist.science technical summary), section 2.1 (LoRA-SVD
linear projection).  The weight is parameterized as W = W_res + beta L2 L1; the
compact principal subspace L2 L1 is kept in BF16 while the main residual W_res is
computed in NVFP4; the low-rank branch is constrained by Cholesky-QR in the
backward pass so its updates stay in the principal subspace; every 2048 steps the
subspace is realigned by a randomized SVD.

The summary prints no equations beyond the parameterization.  Readings (each
the plainest one the text supports):

* L1 (L2 L1's branch): L2 is m x k and L1 is k x n, kept as fp32 masters and
  used in bf16 (round to nearest even) in every product; the branch products
  accumulate in high precision (fp64 here).  With Q(.) the NVFP4 quantizer:
      forward         Y  = Q(X) Q(W_res) + beta (X bf16(L2)) bf16(L1)
      input gradient  dX = Q(D) Q(W_res)^T + beta (D bf16(L1)^T) bf16(L2)^T
      residual grad   dW_res = Q(X^T) Q(D^T)^T          (plain NVFP4 GeMM)
      branch grads    dL2 = beta X^T (D bf16(L1)^T),  dL1 = beta (X bf16(L2))^T D
  i.e. the exact gradients of the forward expression with the quantizer treated
  as the identity in the backward pass (straight-through), X and D in bf16.
* L2 (the Cholesky-QR constraint): after an update, L2 = Q R by CholQR,
  then L2 <- Q and L1 <- R L1.  The product L2 L1, hence W, is unchanged, and L2
  keeps orthonormal columns: the branch stays an orthonormal basis of the
  principal subspace times its coefficients.
* L3 (realignment): W_eff = W_res + beta L2 L1; its rank-k split comes from the
  library's randomized decomposition (Metis refresh and per-step factors, every
  row kept) of bf16(W_eff): W_eff ~ U S V^T; then L2 <- U, L1 <- diag(S / beta)
  V^T and W_res <- W_eff - beta L2 L1, so W is unchanged.

Pins (tests/test_oracle_lora_svd.py): bf16 rounding against torch's conversion
and hand-checked ties; beta = 0 reduces the product to the plain NVFP4 GeMM
written out element by element; a k = 1 all-ones branch gives beta times the row
sums of M (closed form); the branch gradients against central finite
differences of the scalar <D, Y>; the constraint against numpy.linalg.qr up to
column signs and its invariants; the realignment preserves W, returns an
orthonormal L2, and on an exactly rank-k W_eff leaves W_res ~ 0 with the singular
values of numpy.linalg.svd.
"""

import numpy as np

from . import decompose, linalg


def bf16_round(x):
    """Round fp32 values to bfloat16 (8 significant bits), nearest-even, as floats.

    Written from the definition: keep the upper 16 bits of the fp32 pattern,
    adding half an ulp of the kept part (0x7FFF) plus the kept part's lowest
    bit, so that exact halves go to the even neighbour."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def branch_input(which, M, L2, L1):
    """T = M bf16(L2) (which 0) or M bf16(L1)^T (which 1): the branch's first product."""
    M = np.asarray(M, dtype=np.float64)
    if which == 0:
        return M @ bf16_round(L2)
    if which == 1:
        return M @ bf16_round(L1).T
    raise ValueError("which must be 0 or 1")


def lora_linear(which, A_hat, B_hat, M, L2, L1, beta):
    """One product with the branch, from the decoded NVFP4 operands.

    which 0 (forward):        C = A_hat B_hat^T + beta (M bf16(L2)) bf16(L1)
    which 1 (input gradient): C = A_hat B_hat^T + beta (M bf16(L1)^T) bf16(L2)^T
    A_hat: p x K, B_hat: q x K (the K-major decoded operands), M: p x K.
    Returns (C, T) with T = M bf16(L2) or M bf16(L1)^T (p x k)."""
    A_hat = np.asarray(A_hat, dtype=np.float64)
    B_hat = np.asarray(B_hat, dtype=np.float64)
    T = branch_input(which, M, L2, L1)
    branch = T @ bf16_round(L1) if which == 0 else T @ bf16_round(L2).T
    return A_hat @ B_hat.T + beta * branch, T


def branch_grad(M, T, beta):
    """beta M^T T: dL2 = branch_grad(X, D bf16(L1)^T), dL1^T = branch_grad(D, X bf16(L2))."""
    return beta * (np.asarray(M, dtype=np.float64).T @ np.asarray(T, dtype=np.float64))


def constrain(L2, L1):
    """CholQR of L2 (linalg.cholqr, dependent columns dropped): returns (Q, R L1)."""
    Q, R, _ = linalg.cholqr(L2)
    return Q, R @ np.asarray(L1, dtype=np.float64)


def realign(W_res, L2, L1, beta, k, s, seed, operand_id, step, l_k=None):
    """Returns (W_res_new, L2_new, L1_new, S) per reading L3."""
    W_eff = np.asarray(W_res, dtype=np.float64) + beta * (np.asarray(L2, dtype=np.float64) @
                                                         np.asarray(L1, dtype=np.float64))
    m = W_eff.shape[0]
    Wb = bf16_round(W_eff.astype(np.float32))
    basis = decompose.refresh_basis(Wb, k, s, m if l_k is None else l_k, seed, operand_id, step)
    U, S, V = decompose.step_factors(Wb, basis["V"])
    L2n = U
    L1n = (S / beta)[:, None] * V.T
    return W_eff - beta * (L2n @ L1n), L2n, L1n, S
