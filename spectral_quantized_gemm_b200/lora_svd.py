"""LoRA-SVD linear layer for PyTorch training, on libmetis.

``LoRASVDLinear`` computes ``Y = X W`` (X: tokens x in_features, W: in_features x
out_features) with the weight parameterized as ``W = W_res + beta L2 L1``.  Method:
"Full-Stack FP4: stable LLM pretraining with quantized projections, optimizer and
attention" (gist.science technical summary), section 2.1 (LoRA-SVD linear
projection): the compact principal subspace ``L2 L1`` is kept in BF16 while the main
residual ``W_res`` is computed in NVFP4; updates of the low-rank branch are held in the
principal subspace by a Cholesky-QR constraint; the subspace is realigned by a
randomized SVD every 2048 steps.

Every product runs in libmetis:
  forward   Y  = Q(X) Q(W_res) + beta (X L2) L1          (metis_lora_linear, which 0)
  backward  dX = Q(dY) Q(W_res)^T + beta (dY L1^T) L2^T  (metis_lora_linear, which 1)
            dW_res = Q(X^T) Q(dY^T)^T                     (metis_gemm_nvfp4)
            dL2 = beta X^T (dY L1^T), dL1 = beta (X L2)^T dY   (metis_lora_branch_grad)
Q is the NVFP4 quantizer with the decode tensor scale chosen on the device; the
gradient dY is quantized with stochastic rounding.  ``W_res``, ``L2`` and ``L1`` are fp32
``nn.Parameter`` masters updated by any torch optimizer; after each optimizer step call
``post_step()``, which applies the Cholesky-QR constraint (metis_lora_constrain) and,
every ``realign_every`` steps, the realignment (metis_lora_realign).  The first forward
pass realigns the initial weight into its rank-k branch and residual.

Shapes: tokens, in_features and out_features must be multiples of 256; 1 <= k <= 64.
There is no CPU path: the layer needs libmetis on a CUDA device.
"""

import math

import torch

from . import Factors, Nvfp4
from .linear import _shared_context, default_rank


class _LoRASVDFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, W_res, L2, L1, layer):
        y, saved = layer._forward(x.to(torch.bfloat16).contiguous())
        ctx.layer, ctx.saved = layer, saved
        return y

    @staticmethod
    def backward(ctx, dy):
        dx, dW, dL2, dL1 = ctx.layer._backward(dy, ctx.saved)
        ctx.saved = None
        return dx, dW, dL2, dL1, None


class LoRASVDLinear(torch.nn.Module):
    """``Y = X (W_res + beta L2 L1)`` with NVFP4 residual GeMMs and a bf16 rank-k branch.

    Args:
        in_features, out_features: sizes (multiples of 256).
        k: rank of the branch (default: 1.5% of the hidden size, as ``MetisLinear``).
        beta: branch scale.
        realign_every: optimizer steps between randomized-SVD realignments.
        s: oversampling of the randomized decomposition used by the realignment.
        seed: seed of the realignment's sketch and of the stochastic rounding of dY.
    """

    def __init__(self, in_features, out_features, k=None, beta=1.0, realign_every=2048, s=8, seed=0,
                 device=None, dtype=torch.float32):
        super().__init__()
        if in_features % 256 or out_features % 256:
            raise ValueError("in_features and out_features must be multiples of 256")
        if not (math.isfinite(beta) and beta != 0.0):
            raise ValueError("beta must be finite and nonzero")
        self.in_features, self.out_features = int(in_features), int(out_features)
        self.k = default_rank(in_features, out_features) if k is None else int(k)
        if not 1 <= self.k <= 64:
            raise ValueError("k must be in [1, 64]")
        self.beta, self.realign_every, self.s, self.seed = float(beta), int(realign_every), int(s), int(seed)
        self.W_res = torch.nn.Parameter(torch.empty(in_features, out_features, device=device, dtype=dtype))
        self.L2 = torch.nn.Parameter(torch.zeros(in_features, self.k, device=device, dtype=dtype))
        self.L1 = torch.nn.Parameter(torch.zeros(self.k, out_features, device=device, dtype=dtype))
        bound = 1.0 / math.sqrt(in_features)
        with torch.no_grad():
            self.W_res.uniform_(-bound, bound)
        self.step = 0
        self.aligned = False

    def get_extra_state(self):
        return {"step": self.step, "aligned": self.aligned}

    def set_extra_state(self, state):
        self.step, self.aligned = int(state["step"]), bool(state["aligned"])

    def extra_repr(self):
        return (f"in_features={self.in_features}, out_features={self.out_features}, k={self.k}, "
                f"beta={self.beta}, realign_every={self.realign_every}")

    # -- optimizer-side maintenance ----------------------------------------------------
    @torch.no_grad()
    def realign(self):
        """W_eff = W_res + beta L2 L1 -> L2 = U, L1 = S V^T / beta, W_res = W_eff - beta L2 L1."""
        lib, lock = _shared_context(self.W_res.device)
        m, n = self.in_features, self.out_features
        with lock:
            f = Factors(m, n, self.k, device=self.W_res.device)
            Wb = torch.empty(m, n, dtype=torch.bfloat16, device=self.W_res.device)
            lib.lora_realign(self.W_res.data, self.L2.data, self.L1.data, self.beta, f, Wb, s=self.s, l_k=m,
                             seed=self.seed, operand_id=1, step=self.step)
        self.aligned = True

    @torch.no_grad()
    def post_step(self):
        """Call after each optimizer step: the Cholesky-QR constraint on the branch, and
        the realignment every ``realign_every`` steps."""
        lib, lock = _shared_context(self.W_res.device)
        with lock:
            lib.lora_constrain(self.L2.data, self.L1.data)
        self.step += 1
        if self.step % self.realign_every == 0:
            self.realign()

    # -- the products ------------------------------------------------------------------
    def forward(self, x):
        if x.shape[-1] != self.in_features:
            raise ValueError(f"expected last dimension {self.in_features}, got {x.shape[-1]}")
        if not self.aligned:
            self.realign()
        lead = x.shape[:-1]
        y = _LoRASVDFn.apply(x.reshape(-1, self.in_features), self.W_res, self.L2, self.L1, self)
        return y.reshape(*lead, self.out_features)

    def _quantize(self, lib, M, op_id, rounding):
        rows, cols = M.shape
        row, col = Nvfp4(rows, cols, M.device), Nvfp4(cols, rows, M.device)
        lib.residual_quantize_nvfp4(M, None, rowwise=row, colwise=col, rounding=rounding, seed=self.seed,
                                    operand_id=op_id, step=self.step, tensor_scale=0.0)
        return row, col

    def _forward(self, x):
        rows = x.shape[0]
        if rows % 256:
            raise ValueError(f"the number of tokens ({rows}) must be a multiple of 256")
        lib, lock = _shared_context(x.device)
        with lock:
            xr, xc = self._quantize(lib, x, 0, 0)
            wr, wc = self._quantize(lib, self.W_res.detach().to(torch.bfloat16).contiguous(), 1, 0)
            y = torch.empty(rows, self.out_features, dtype=torch.bfloat16, device=x.device)
            T_x = torch.empty(rows, self.k, dtype=torch.float32, device=x.device)
            lib.lora_linear(0, xr, wc, x, self.L2.detach(), self.L1.detach(), self.beta, y, T=T_x)
        return y, (x, xc, wr, T_x)

    def _backward(self, dy, saved):
        x, xc, wr, T_x = saved
        dy = dy.to(torch.bfloat16).contiguous()
        rows = dy.shape[0]
        lib, lock = _shared_context(dy.device)
        with lock:
            dr, dc = self._quantize(lib, dy, 2, 1)
            dx = torch.empty(rows, self.in_features, dtype=torch.bfloat16, device=dy.device)
            T_d = torch.empty(rows, self.k, dtype=torch.float32, device=dy.device)
            lib.lora_linear(1, dr, wr, dy, self.L2.detach(), self.L1.detach(), self.beta, dx, T=T_d)
            dW = torch.empty(self.in_features, self.out_features, dtype=torch.float32, device=dy.device)
            lib.gemm_nvfp4(xc, dc, self.out_features, dW)
            dL2 = torch.empty(self.in_features, self.k, dtype=torch.float32, device=dy.device)
            dL1 = torch.empty(self.k, self.out_features, dtype=torch.float32, device=dy.device)
            lib.lora_branch_grad(x, T_d, self.beta, dL2)
            lib.lora_branch_grad(dy, T_x, self.beta, dL1, transpose_out=True)
        return dx, dW, dL2, dL1
