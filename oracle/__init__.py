"""CPU oracle for the Metis spectral-domain W4A4G4 linear layer.

This package is TEST INFRASTRUCTURE. It is a plain, slow, fp64 restatement of
the method, written from the description of Metis ("Metis: Training LLMs with
FP4 Quantization", papernotes.org notes on the ICLR 2026 paper) and checked
against closed forms, invariants and textbook routines in ``tests/``.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The CUDA library
(``spectral_quantized_gemm_b200``) never imports it and shares no code with
it; the only thing both sides consume is the seeded input generator in
``workloads/``, which holds none of the method's arithmetic.

Modules, in the order the method uses them:

* ``philox``    -- Philox4x32-10 counter generator and the stream layout
                   (row sampling, Gaussian test matrix, stochastic rounding).
* ``formats``   -- E2M1 and E4M3 tables; encoders by exhaustive nearest search.
* ``nvfp4``     -- NVFP4 block quantizer Q_b (16-element blocks, E4M3 scale,
                   round-to-nearest or stochastic rounding).
* ``linalg``    -- CholQR and one-sided Jacobi SVD in fp64.
* ``decompose`` -- row sampling, sketch, subspace refresh, per-step factors,
                   residual M_R = M - U S V^T.
* ``metis``     -- the mixed-precision product for the forward, dX and dW
                   GEMMs, and the end-to-end layer.
* ``lora_svd``  -- the LoRA-SVD linear projection W = W_res + beta L2 L1
                   ("Full-Stack FP4" technical summary, section 2.1): the branch
                   product, its gradients, the Cholesky-QR constraint and the
                   randomized-SVD realignment.

Parity status of every function is listed in its module header.  Nothing in
this package is "parity unpinned" except where a header says so explicitly.
"""

from . import philox, formats, nvfp4, linalg, decompose, metis, lora_svd  # noqa: F401
