"""Sampling-ratio sweep and spectral-distortion diagnostics on the GPU kernels.

The alignment of the sampled-row basis with the all-rows basis is compared with the
same quantity from the oracle's decomposition; the plain-NVFP4 per-direction errors
with those of the oracle's quantizer (bit-exact decode, so they are equal); and on
channel-spiked data Metis's errors along the small singular directions are below plain
NVFP4's (the distortion the method's background section describes).
"""

import numpy as np
import pytest
import torch

from oracle import decompose, linalg, nvfp4
from workloads import synth

pytestmark = pytest.mark.gpu


def _matrix(rows, cols, n_spike, rho, seed):
    A = synth.anisotropic(rows, cols, n_spike, 50.0, rho, np.random.default_rng(seed), "channels")
    return synth.to_bf16(A)


def test_sampling_alignment_matches_the_oracle(ctx, metis_lib):
    from spectral_quantized_gemm_b200 import analysis
    Mt = _matrix(1024, 512, 20, 0.9, 21)
    k, s = 16, 8
    res = analysis.sampling_alignment(ctx, Mt.cuda(), k, s, [0.03, 0.1, 0.5], seeds=(0, 1))
    Md = Mt.double().numpy()
    assert [r["l_k"] for r in res] == [31, 103, 512]
    for r in res:
        al, en = [], []
        for sd in (0, 1):
            Vf = decompose.refresh_basis(Md, k, s, 1024, sd, 0, 0)["V"]
            Vs = decompose.refresh_basis(Md, k, s, r["l_k"], sd, 0, 0)["V"]
            al.append(linalg.principal_cosines(Vs, Vf).mean())
            en.append(np.linalg.norm(Md @ Vs) ** 2 / np.linalg.norm(Md @ Vf) ** 2)
        assert abs(np.mean(al) - r["alignment"]) < 2e-3, (r, al)
        assert abs(np.mean(en) - r["energy"]) < 1e-4, (r, en)
        assert r["energy"] <= 1.0 + 1e-3      # the all-rows basis captures (nearly) the most
    assert res[-1]["alignment"] >= res[0]["alignment"] - 1e-3     # more rows, no worse
    assert ctx.poll_device_status() == 0


def test_spectral_distortion(ctx, metis_lib):
    from spectral_quantized_gemm_b200 import analysis
    Mt = _matrix(1024, 512, 10, 0.9, 22)
    d = analysis.spectral_distortion(ctx, Mt.cuda(), k=16, s=8, l_k=1024, rounding=0)
    assert ctx.poll_device_status() == 0
    Md = Mt.double().numpy()
    codes, scales = nvfp4.quantize_oriented(Md.astype(np.float32), "row")
    sig, err, leak = analysis.direction_errors(Md, nvfp4.dequantize_blocks(codes, scales, 1.0))
    assert np.allclose(d["sigma"], sig)
    assert np.allclose(d["plain"], err, rtol=1e-9, atol=1e-12)
    assert np.allclose(d["plain_leak"], leak, rtol=1e-9, atol=1e-12)
    n = len(sig)
    tail = slice(n // 2, n)          # the small singular directions
    assert np.median(d["metis"][tail]) < np.median(d["plain"][tail])
    assert np.median(d["metis_leak"][tail]) < np.median(d["plain_leak"][tail])
