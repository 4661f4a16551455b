"""Seeded synthetic inputs shaped like the Metis workloads.

Shared by the CUDA path's tests and benchmark and by the oracle's tests.  It
holds no arithmetic of the method: it only draws anisotropic bf16 matrices
and names the workload configurations.
"""

from .synth import CONFIGS, anisotropic, operand_matrix, perturbed, n_spikes  # noqa: F401
