"""Run one stage of the Metis layer a few times on one synthetic operand, for a profiler.

    python spectral_quantized_gemm_b200/profile_case.py {resquant,decompose,step,gemm} \
        [--rows R] [--cols C] [--k K] [--inner K2] [--fold F] [--bf16] [--reps N]

``resquant``: the fused residual NVFP4 quantizer (both orientations) of an
R x C bf16 operand with rank-K factors.  ``decompose``: the per-step factor
update (P = M V, CholQR, small SVD) of the same operand.  ``step``: both.
``gemm``: the fused FP4 GeMM C (R x C) = A (R x K2) B^T (C x K2) plus a rank fold of
width F, on plain NVFP4 operands (fp32 output, or bf16 with --bf16).
A profiler filters the launches by kernel name; this driver only issues them.
"""

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import spectral_quantized_gemm_b200 as sq  # noqa: E402
from workloads import synth  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("stage", choices=["resquant", "decompose", "step", "gemm"])
    ap.add_argument("--rows", type=int, default=8192)
    ap.add_argument("--cols", type=int, default=14336)
    ap.add_argument("--k", type=int, default=64)
    ap.add_argument("--s", type=int, default=8)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--inner", type=int, default=4096)
    ap.add_argument("--fold", type=int, default=256)
    ap.add_argument("--bf16", action="store_true")
    a = ap.parse_args()
    if a.stage == "gemm":
        return gemm_case(a)
    cfg = synth.scaled_config("llama3_8b_mlp_up", l=a.rows, m=a.cols, n=a.cols)
    M = synth.operand_matrix(cfg, "X").cuda()
    ctx = sq.Context(0)
    f = ctx.new_factors(a.rows, a.cols, a.k)
    ctx.decompose(M, k=a.k, s=a.s, l_k=min(a.rows, 82), seed=1, operand_id=0, refresh=True, step=0, factors=f)
    row, col = ctx.new_nvfp4(a.rows, a.cols), ctx.new_nvfp4(a.cols, a.rows)
    for t in range(1, a.reps + 1):
        if a.stage in ("decompose", "step"):
            ctx.decompose(M, k=a.k, s=a.s, l_k=min(a.rows, 82), seed=1, operand_id=0, refresh=False, step=t,
                          factors=f)
        if a.stage in ("resquant", "step"):
            ctx.residual_quantize_nvfp4(M, f, row, col, rounding=1, seed=1, operand_id=0, step=t)
    torch.cuda.synchronize()
    status = ctx.poll_device_status()
    print(f"{a.stage}: {a.rows}x{a.cols} k={a.k} reps={a.reps} device_status={status}")
    sys.exit(1 if status else 0)


def gemm_case(a):
    ctx = sq.Context(0)
    g = torch.Generator(device="cuda").manual_seed(0)
    A = torch.randn(a.rows, a.inner, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(a.cols, a.inner, device="cuda", generator=g).to(torch.bfloat16)
    qa, qb = ctx.new_nvfp4(a.rows, a.inner), ctx.new_nvfp4(a.cols, a.inner)
    ctx.residual_quantize_nvfp4(A, None, rowwise=qa)
    ctx.residual_quantize_nvfp4(B, None, rowwise=qb)
    Fa = Fb = None
    if a.fold:
        Fa = (0.01 * torch.randn(a.rows, a.fold, device="cuda", generator=g)).to(torch.bfloat16)
        Fb = (0.01 * torch.randn(a.cols, a.fold, device="cuda", generator=g)).to(torch.bfloat16)
    C = torch.empty(a.rows, a.cols, device="cuda", dtype=torch.bfloat16 if a.bf16 else torch.float32)
    for _ in range(a.reps):
        ctx.gemm_nvfp4(qa, qb, a.cols, C, Fa, Fb)
    torch.cuda.synchronize()
    status = ctx.poll_device_status()
    print(f"gemm: {a.rows}x{a.cols}x{a.inner} fold={a.fold} bf16={a.bf16} reps={a.reps} device_status={status}")
    sys.exit(1 if status else 0)


if __name__ == "__main__":
    main()
