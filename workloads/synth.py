"""Anisotropic synthetic matrices and the workload table.

The Metis notes ("Metis: Training LLMs with FP4 Quantization", 研究背景 /
核心矛盾 and 关键发现) observe that fewer than 3% of singular values dominate
the spectra of weights, activations and gradients, with a long bulk tail.
The experiments (主实验: LLaMA-3 8B and GPT-2 on DCLM) need trained weights and
data that are not available here, so every matrix is synthetic:

    M = P diag(sigma) Q^T + N(0, 1)

with P Gaussian / sqrt(rows), sigma_i = sigma0 * rho^i * sqrt(rows), drawn in
fp64 from numpy's default_rng seeded by (seed, operand) and rounded to bf16.
Q (cols x n_spike) has orthonormal columns of one of two kinds:

* "dense": the orthonormal factor of a Gaussian (the tiny workload);
* "channels": distinct columns of the identity, so each spike lives on one
  hidden dimension (an outlier channel).  This is the reading of "2% spike
  dims" for the layer-shaped workloads; it produces the long-tailed entry
  distribution the notes describe (a few large values set the block maximum
  and crush the small ones).

The number of spikes is round(0.02 * min(rows, cols)) unless a configuration
fixes it.

The layer shapes are those of GPT-2 small's MLP up-projection and LLaMA-3
8B's MLP up- and down-projections at 8192 tokens, plus a long-token stress
shape; the ranks follow the 1.5% rule (训练策略) and l_k the 1% row sample
(关键设计 2 / 消融).
"""

import numpy as np
import torch

OPERAND_IDS = {"X": 0, "W": 1, "D": 2}


def n_spikes(rows, cols):
    return int(round(0.02 * min(rows, cols)))


def anisotropic(rows, cols, n_spike, sigma0, rho, rng, directions="dense"):
    """fp64 rows x cols matrix: spiked low-rank part plus N(0,1) bulk."""
    out = rng.standard_normal((rows, cols))
    if n_spike > 0:
        P = rng.standard_normal((rows, n_spike)) / np.sqrt(rows)
        sigma = sigma0 * rho ** np.arange(n_spike) * np.sqrt(rows)
        if directions == "dense":
            Q, _ = np.linalg.qr(rng.standard_normal((cols, n_spike)))
            out += (P * sigma[None, :]) @ Q.T
        elif directions == "channels":
            channels = rng.choice(cols, size=n_spike, replace=False)
            out[:, channels] += P * sigma[None, :]
        else:
            raise ValueError(directions)
    return out


def to_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


CONFIGS = {
    # one metis_linear_fwd on 256 x 256 operands, six spikes
    "tiny_fwd": dict(l=256, m=256, n=256, k=4, s=4, l_k=32, sigma0=40.0, rho=0.8, seed=0,
                     spikes={"X": 6, "W": 6, "D": 6}, directions="dense", rounding="rn", fwd_only=True,
                     refresh_every=8, steps=1),
    # GPT-2 small MLP up-projection, 8 sequences x 1024 tokens
    "gpt2_small_mlp_up": dict(l=8192, m=768, n=3072, k=12, s=8, l_k=82, sigma0=50.0, rho=0.9,
                              seed=1, spikes=None, directions="channels", rounding="sr", fwd_only=False,
                              refresh_every=8, steps=1),
    # LLaMA-3 8B MLP up-projection, 8192 tokens
    "llama3_8b_mlp_up": dict(l=8192, m=4096, n=14336, k=64, s=8, l_k=82, sigma0=50.0, rho=0.9,
                             seed=2, spikes=None, directions="channels", rounding="sr", fwd_only=False,
                             refresh_every=8, steps=1),
    # LLaMA-3 8B down-projection, one decomposition reused over 8 perturbed steps
    "llama3_8b_down_reuse": dict(l=8192, m=14336, n=4096, k=64, s=8, l_k=82, sigma0=50.0,
                                 rho=0.9, seed=3, spikes=None, directions="channels", rounding="sr", fwd_only=False,
                                 refresh_every=8, steps=8, perturb=1e-2),
    # long-token stress, 16 sequences x 4096 tokens, refresh every step and every 8th step
    "long_token_stress": dict(l=65536, m=4096, n=4096, k=64, s=8, l_k=655, sigma0=50.0,
                              rho=0.9, seed=4, spikes=None, directions="channels", rounding="sr", fwd_only=False,
                              refresh_every=1, steps=1),
}


def operand_shape(cfg, name):
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    return {"X": (l, m), "W": (m, n), "D": (l, n)}[name]


def operand_matrix(cfg, name, as_numpy=False):
    """The bf16 matrix of operand X, W or D of a configuration (CPU tensor)."""
    rows, cols = operand_shape(cfg, name)
    spikes = cfg["spikes"][name] if cfg.get("spikes") else n_spikes(rows, cols)
    rng = np.random.default_rng([cfg["seed"], OPERAND_IDS[name]])
    M = anisotropic(rows, cols, spikes, cfg["sigma0"], cfg["rho"], rng, cfg.get("directions", "dense"))
    t = to_bf16(M)
    return t.double().numpy() if as_numpy else t


def batch_matrix(cfg, name, batch):
    """Operand of training batch ``batch`` (bf16, CPU): a new draw of the tokens.

    The layer's persistent structure -- the spike directions (outlier channels or
    dense directions) and their magnitudes -- comes from a generator seeded by
    (seed, operand); the token content -- the spike coefficients P and the N(0, 1)
    bulk -- from one seeded by (seed, operand, batch).  So consecutive batches share
    their dominant subspace, as the notes observe for activations and gradients
    (关键设计 3), while no two batches have the same values.
    """
    rows, cols = operand_shape(cfg, name)
    n_spike = cfg["spikes"][name] if cfg.get("spikes") else n_spikes(rows, cols)
    srng = np.random.default_rng([cfg["seed"], OPERAND_IDS[name], 7])
    crng = np.random.default_rng([cfg["seed"], OPERAND_IDS[name], 100 + int(batch)])
    out = crng.standard_normal((rows, cols))
    if n_spike > 0:
        sigma = cfg["sigma0"] * cfg["rho"] ** np.arange(n_spike) * np.sqrt(rows)
        P = crng.standard_normal((rows, n_spike)) / np.sqrt(rows)
        if cfg.get("directions", "dense") == "dense":
            Q, _ = np.linalg.qr(srng.standard_normal((cols, n_spike)))
            out += (P * sigma[None, :]) @ Q.T
        else:
            channels = srng.choice(cols, size=n_spike, replace=False)
            out[:, channels] += P * sigma[None, :]
    return to_bf16(out)


def perturbed(cfg, name, base, step):
    """base + perturb * rms(base) * N(0,1), fresh noise per step (bf16)."""
    rng = np.random.default_rng([cfg["seed"], OPERAND_IDS[name], 1000 + int(step)])
    b = base.double().numpy()
    rms = float(np.sqrt(np.mean(b * b)))
    noisy = b + cfg.get("perturb", 0.0) * rms * rng.standard_normal(b.shape)
    return to_bf16(noisy)


def scaled_config(name, l=None, m=None, n=None, **over):
    """A copy of a configuration with other sizes (for small parity cases)."""
    cfg = dict(CONFIGS[name])
    for key, val in (("l", l), ("m", m), ("n", n)):
        if val is not None:
            cfg[key] = val
    cfg.update(over)
    return cfg
