"""Run one stage of the Metis layer a few times on one synthetic operand, for a profiler.

    python spectral_quantized_gemm_b200/profile_case.py {resquant,decompose,step} \
        [--rows R] [--cols C] [--k K] [--reps N]

``resquant``: the fused residual NVFP4 quantizer (both orientations) of an
R x C bf16 operand with rank-K factors.  ``decompose``: the per-step factor
update (P = M V, CholQR, small SVD) of the same operand.  ``step``: both.
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
    ap.add_argument("stage", choices=["resquant", "decompose", "step"])
    ap.add_argument("--rows", type=int, default=8192)
    ap.add_argument("--cols", type=int, default=14336)
    ap.add_argument("--k", type=int, default=64)
    ap.add_argument("--s", type=int, default=8)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
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


if __name__ == "__main__":
    main()
