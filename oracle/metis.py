"""The Metis mixed-precision product and the W4A4G4 linear layer.

Source: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
关键设计 1: with X = A_k Lambda_k B_k^T + X_R and W = U_k S_k V_k^T + W_R the
forward GeMM is

    Y_hat = (Q(A_k) Lambda_k Q(B_k^T) + Q(X_R)) (Q(U_k) S_k Q(V_k^T) + Q(W_R))

where Q_b acts on every matrix except the singular values.  整体框架 embeds
the same split in every forward and backward GeMM (W4A4G4); the pages print
no backward formula, so (reading R13) the two backward GeMMs apply the same
split to both of their operands:

    dX_hat = D_hat W_hat^T          dW_hat = X_hat^T D_hat

Each operand hat is formed from its own quantized pieces.  The residual is
quantized with 16-blocks along the contraction dimension of the GeMM that
uses it (reading R5), so every residual has two quantizations: row-wise
(blocks along columns) and column-wise (blocks along rows).  The factors are
quantized once, with blocks along their long dimension, and with a
power-of-two per-tensor decode scale (reading R1).

The oracle evaluates each GeMM as the plain definition: the dense fp64
operand hats, then one fp64 matrix product (no intermediate is re-quantized,
reading R14).

Pins (tests/test_oracle_metis.py): k = 0 equals plain NVFP4 GeMM; with
quantization replaced by the identity the product equals the exact X W; the
four-term expansion agrees with the dense form; on anisotropic inputs the
Metis error against the exact X W is below plain-NVFP4 error.
"""

import numpy as np

from . import decompose, nvfp4, philox

FACTOR_SCALE_DIVISOR = np.float32(6.0 * 448.0)


def factor_tensor_scale(F):
    """Smallest power of two g with amax(F) / (6 * 448 * g) <= 1 (g = 1 if F == 0)."""
    amax = np.float32(np.max(np.abs(np.asarray(F, dtype=np.float32)))) if np.size(F) else np.float32(0)
    if amax == 0:
        return 1.0
    t = np.float32(amax / FACTOR_SCALE_DIVISOR)
    mant, expo = np.frexp(np.float64(t))      # t = mant * 2^expo, mant in [0.5, 1)
    return float(2.0 ** (expo - 1)) if mant == 0.5 else float(2.0 ** expo)


def quantize_factor(F, seed=0, operand_id=0, sub=philox.SR_SUB_LEFT, step=0, rounding="rn"):
    """Quantize a long x k factor with blocks along its long dimension.

    Returns (codes, scales, g) for the k x long transposed view.
    """
    F = np.asarray(F, dtype=np.float32)
    g = factor_tensor_scale(F)
    codes, scales = nvfp4.quantize_oriented(F, "col", g=g, rounding=rounding, seed=seed,
                                            operand_id=operand_id, step=step, sr_sub=sub)
    return codes, scales, g


def prepare_operand(M, V, seed=0, operand_id=0, step=0, rounding="rn", g_res=1.0, k=None):
    """Per-step work for one operand on the reused basis V (None or k == 0: plain NVFP4).

    Returns a dict with the unquantized factors, the fp32 residual, both
    residual quantizations and the quantized factors.
    """
    M = np.asarray(M, dtype=np.float64)
    op = {"shape": M.shape}
    if V is None or (k is not None and k == 0) or np.asarray(V).shape[1] == 0:
        op["U"] = op["V"] = op["S"] = None
        R = M.astype(np.float32)
    else:
        U, S, Vn = decompose.step_factors(M, V)
        op["U"], op["S"], op["V"] = U, S, Vn
        R = decompose.residual(M, U, S, Vn)
        op["Uq"] = quantize_factor(U.astype(np.float32), seed, operand_id, philox.SR_SUB_LEFT, step, rounding)
        op["Vq"] = quantize_factor(Vn.astype(np.float32), seed, operand_id, philox.SR_SUB_RIGHT, step, rounding)
    op["R"] = R
    for orient in ("row", "col"):
        codes, scales = nvfp4.quantize_oriented(R, orient, g=g_res, rounding=rounding, seed=seed,
                                                operand_id=operand_id, step=step)
        op[orient] = (codes, scales, g_res)
    return op


def dequant_residual(op, orientation):
    codes, scales, g = op[orientation]
    D = nvfp4.dequantize_blocks(codes, scales, g)
    return D if orientation == "row" else D.T


def dequant_factor(q):
    codes, scales, g = q
    return nvfp4.dequantize_blocks(codes, scales, g).T      # long x k


def operand_hat(op, orientation):
    """Dense fp64 Q(U) S Q(V)^T + Q(M_R) for one residual orientation."""
    hat = dequant_residual(op, orientation)
    if op.get("U") is not None:
        Uq = dequant_factor(op["Uq"])
        Vq = dequant_factor(op["Vq"])
        S = np.asarray(op["S"], dtype=np.float64)
        hat = hat + (Uq * S[None, :]) @ Vq.T
    return hat


def linear_fwd(opX, opW):
    return operand_hat(opX, "row") @ operand_hat(opW, "col")


def linear_bwd(opX, opW, opD):
    dX = operand_hat(opD, "row") @ operand_hat(opW, "row").T
    dW = operand_hat(opX, "col").T @ operand_hat(opD, "col")
    return dX, dW


def fold_terms(opA_hat_parts, opB_hat_parts):
    """Four-term expansion of (L_A S_A R_A^T + A_R)(L_B S_B R_B^T + B_R), for cross-checks.

    Each argument is (L, S, R, Resid) with dense fp64 pieces.
    """
    LA, SA, RA, AR = opA_hat_parts
    LB, SB, RB, BR = opB_hat_parts
    main = AR @ BR
    TA = (SA[:, None] * RA.T) @ (BR + (LB * SB[None, :]) @ RB.T)
    TB = AR @ (LB * SB[None, :])
    return main + LA @ TA + TB @ RB.T
