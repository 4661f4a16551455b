"""Diagnostics of the decomposition and the quantizer, run on the library's kernels.

Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes).

* ``sampling_alignment``: key design 2 decomposes an activation or gradient from a
  sample of about 1% of its token rows, and the notes report that the subspace found
  this way aligns with the full-batch one to about 0.9.  Here the basis V_k of the
  randomized decomposition from ``l_k = ratio * rows`` sampled rows is compared with
  the basis from all rows (the same kernels with l_k = rows): the alignment is the
  mean of the principal cosines between the two k-dimensional column spans (1 for
  the same subspace), and the smallest principal cosine is reported beside it.  As
  near-degenerate trailing directions make single cosines ill-defined, the energy ratio
  ||M V_sampled||_F^2 / ||M V_all||_F^2 (the share of what the all-rows basis captures
  that the sampled basis captures too) is reported as well.
* ``spectral_distortion``: the background section argues that block-wise FP4 rounds
  small values to zero and distorts the small singular components of a matrix.  For
  each singular triple (sigma_i, u_i, v_i) of M (exact SVD in fp64 on the host) this
  measures the error of the quantized matrix M_hat along that direction,
  |u_i^T (M_hat - M) v_i| / sigma_i, and the leakage ||(M_hat - M) v_i|| / sigma_i,
  for plain NVFP4 (M_hat = Q(M)) and for Metis (M_hat = Q(M - U S V^T) + Q(U) S Q(V)^T).
  The quantized matrices are decoded on the device (metis_dequantize_nvfp4).

Run ``python -m spectral_quantized_gemm_b200.analysis`` from the repository root for
the sweep on the synthetic spectra of the layer workloads (``workloads/synth.py``).
The decompositions and quantizations run in libmetis on the GPU; the principal
angles and the per-direction errors are host-side numpy on small outputs.
"""

import math

import numpy as np

from . import Context


def principal_cosines(V1, V2):
    """Cosines of the principal angles between the column spans of V1 and V2
    (orthonormal columns), descending."""
    A = np.asarray(V1, dtype=np.float64)
    B = np.asarray(V2, dtype=np.float64)
    return np.clip(np.linalg.svd(A.T @ B, compute_uv=False), 0.0, 1.0)


def _basis(ctx, M, k, s, l_k, seed, operand_id):
    rows, cols = M.shape
    f = ctx.new_factors(rows, cols, k)
    ctx.decompose(M, k=k, s=s, l_k=l_k, seed=seed, operand_id=operand_id, refresh=True, step=0, factors=f)
    return f.V.double().cpu().numpy()


def sampling_alignment(ctx, M, k, s, ratios, seeds=(0, 1, 2), operand_id=0):
    """Alignment of the sampled-row basis with the all-rows basis at each sampling ratio.

    M: bf16 CUDA matrix (rows x cols).  Returns one dict per ratio with l_k, the mean
    and spread over seeds of the mean principal cosine, and the worst smallest cosine."""
    rows = M.shape[0]
    Md = M.double().cpu().numpy()
    full = [_basis(ctx, M, k, s, rows, sd, operand_id) for sd in seeds]
    full_energy = [np.linalg.norm(Md @ V) ** 2 for V in full]
    out = []
    for ratio in ratios:
        l_k = int(min(rows, max(k + s, math.ceil(ratio * rows))))
        means, mins, energy = [], [], []
        for i, sd in enumerate(seeds):
            Vs = _basis(ctx, M, k, s, l_k, sd, operand_id)
            cos = principal_cosines(Vs, full[i])
            means.append(cos.mean())
            mins.append(cos.min())
            energy.append(np.linalg.norm(Md @ Vs) ** 2 / full_energy[i])
        out.append(dict(ratio=ratio, l_k=l_k, alignment=float(np.mean(means)), spread=float(np.std(means)),
                        min_cosine=float(np.min(mins)), energy=float(np.mean(energy))))
    return out


def _decoded_factor(ctx, q, k):
    """Q(F)^T was stored as NVFP4 with outer padded to 128: decode and keep k rows."""
    return ctx.dequantize_nvfp4(q)[:k].double().cpu().numpy().T


def direction_errors(M, M_hat, n_dirs=None):
    """For the leading n_dirs singular triples (sigma_i, u_i, v_i) of M (fp64 host
    arrays): sigma, |u_i^T (M_hat - M) v_i| / sigma_i and ||(M_hat - M) v_i|| / sigma_i."""
    M = np.asarray(M, dtype=np.float64)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    n = len(S) if n_dirs is None else min(n_dirs, len(S))
    U, S, V = U[:, :n], S[:n], Vt[:n].T
    EV = (np.asarray(M_hat, dtype=np.float64) - M) @ V
    return S, np.abs(np.einsum("ri,ri->i", U, EV)) / S, np.linalg.norm(EV, axis=0) / S


def spectral_distortion(ctx, M, k, s, l_k, n_dirs=None, seed=0, rounding=0):
    """Per-singular-direction error of plain NVFP4 and of Metis on M (bf16 CUDA).

    Returns dict(sigma, plain, metis, plain_leak, metis_leak), arrays over the leading
    n_dirs singular directions (all of them by default)."""
    rows, cols = M.shape
    Md = M.double().cpu().numpy()

    plain = ctx.new_nvfp4(rows, cols)
    ctx.residual_quantize_nvfp4(M, None, rowwise=plain, rounding=rounding, seed=seed, operand_id=0, step=0)
    hat_plain = ctx.dequantize_nvfp4(plain).double().cpu().numpy()

    f = ctx.new_factors(rows, cols, k)
    ctx.decompose(M, k=k, s=s, l_k=l_k, seed=seed, operand_id=0, refresh=True, step=0, factors=f, rounding=rounding)
    res = ctx.new_nvfp4(rows, cols)
    ctx.residual_quantize_nvfp4(M, f, rowwise=res, rounding=rounding, seed=seed, operand_id=0, step=0)
    Uq = _decoded_factor(ctx, f.Uq, k)
    Vq = _decoded_factor(ctx, f.Vq, k)
    Sf = f.S[:k].double().cpu().numpy()
    hat_metis = ctx.dequantize_nvfp4(res).double().cpu().numpy() + (Uq * Sf) @ Vq.T

    out = {}
    for name, hat in (("plain", hat_plain), ("metis", hat_metis)):
        out["sigma"], out[name], out[name + "_leak"] = direction_errors(Md, hat, n_dirs)
    return out


def _main():
    import argparse
    import os
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from workloads import synth

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--ratios", default="0.0025,0.005,0.01,0.02,0.05,0.1")
    ap.add_argument("--seeds", type=int, default=3)
    args = ap.parse_args()
    ratios = [float(r) for r in args.ratios.split(",")]
    ctx = Context()
    seeds = tuple(range(args.seeds))
    print("sampling alignment (mean principal cosine of sampled-row vs all-row V_k, mean over seeds; "
          "energy = ||M V_s||^2 / ||M V_all||^2)")
    for label, rows, cols, rho, directions in (("channel spikes, rho 0.9", 8192, 4096, 0.9, "channels"),
                                               ("channel spikes, rho 0.97", 8192, 4096, 0.97, "channels"),
                                               ("dense spikes, rho 0.9", 8192, 4096, 0.9, "dense")):
        rng = np.random.default_rng(11)
        A = synth.anisotropic(rows, cols, synth.n_spikes(rows, cols), 50.0, rho, rng, directions)
        M = synth.to_bf16(A).cuda()
        for r in sampling_alignment(ctx, M, 64, 8, ratios, seeds):
            print(f"  {label:26s} {rows}x{cols} k=64 ratio {100 * r['ratio']:5.2f}% l_k={r['l_k']:5d}  "
                  f"alignment {r['alignment']:.4f} (+-{r['spread']:.4f})  min cosine {r['min_cosine']:.4f}  "
                  f"energy {r['energy']:.4f}")
    print("spectral distortion: |u_i^T (M_hat - M) v_i| / sigma_i, median over direction groups")
    rng = np.random.default_rng(12)
    A = synth.anisotropic(2048, 1024, synth.n_spikes(2048, 1024), 50.0, 0.9, rng, "channels")
    M = synth.to_bf16(A).cuda()
    d = spectral_distortion(ctx, M, k=16, s=8, l_k=2048, rounding=0)
    n = len(d["sigma"])
    for lo, hi in ((0, 16), (16, 64), (64, 256), (256, n // 2), (n // 2, n)):
        print(f"  directions {lo:4d}-{hi - 1:4d} (sigma {d['sigma'][lo]:9.2f} .. {d['sigma'][hi - 1]:7.2f}): "
              f"plain {np.median(d['plain'][lo:hi]):.4f}  metis {np.median(d['metis'][lo:hi]):.4f}  "
              f"leak plain {np.median(d['plain_leak'][lo:hi]):.4f}  metis {np.median(d['metis_leak'][lo:hi]):.4f}")
    assert ctx.poll_device_status() == 0


if __name__ == "__main__":
    _main()
