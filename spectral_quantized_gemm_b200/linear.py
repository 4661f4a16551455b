"""Drop-in Metis linear layer for PyTorch training.

``MetisLinear`` computes ``Y = X W`` (X: tokens x in_features, W: in_features x
out_features, the notation of the method) with the forward GeMM and both backward
GeMMs (dX = dY W^T, dW = X^T dY) run as the Metis spectral W4A4G4 product inside
libmetis.  Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org
notes): the split of every operand into a rank-k spectral part and an NVFP4
residual is embedded in every forward and backward GeMM (framework section); the
randomized decomposition is refreshed every ``refresh_every`` steps and its basis
reused in between (key design 3 and the training strategy); the rank is 1.5% of the
hidden size and gradients use stochastic rounding (training strategy).

The module keeps an fp32 master weight (an ``nn.Parameter``); each call casts it and
the input to bf16, the layer's input type.  Every operand's NVFP4 decode tensor scale
is chosen on the device from its magnitude (a power of two that puts its largest
entry well inside the E4M3 block-scale range), which gradients need.  Per operand (X, W, dY) it keeps the
reused basis V between calls; everything else of a call (factors, NVFP4 operands)
lives in a per-call slot that the backward pass releases, so several forward passes
may be in flight before their backward passes (gradient accumulation).

Shapes: tokens, in_features and out_features must be multiples of 256.  There is no
CPU path: the layer needs libmetis on a CUDA device.
"""

import math
import threading

import torch

from . import Context, Factors, Nvfp4

_CONTEXTS = {}
_CONTEXT_LOCK = threading.Lock()


def _shared_context(device):
    """One libmetis context per device, shared by every MetisLinear on it (its calls run
    on torch's current stream and are serialized by the returned lock)."""
    with _CONTEXT_LOCK:
        entry = _CONTEXTS.get(device.index)
        if entry is None:
            with torch.cuda.device(device):
                entry = (Context(device.index), threading.Lock())
            _CONTEXTS[device.index] = entry
        return entry


def default_rank(in_features, out_features):
    """1.5% of the hidden size, rounded up to a multiple of 4, at most 64 (the
    training strategy's rank: 64 for 4096, 12 for 768)."""
    return int(min(64, 4 * math.ceil(0.015 * min(in_features, out_features) / 4)))


class _Operand:
    """One operand of one call: factors (sharing nothing with other calls) and its
    row-wise and column-wise NVFP4 residuals."""

    def __init__(self, rows, cols, k, device):
        self.factors = Factors(rows, cols, k, device=device)
        self.row = Nvfp4(rows, cols, device)
        self.col = Nvfp4(cols, rows, device)
        self.struct = Context.operand(self.row, self.col, self.factors)


class _Basis:
    """The reused right basis V of one operand stream (X, W or dY) between refreshes."""

    def __init__(self):
        self.V = None
        self.shape = None


class _MetisLinearFn(torch.autograd.Function):
    # Inputs are the caller's x (any float type) and the master weight; the bf16 casts
    # happen inside, so dW reaches the master weight in fp32 and dX is cast to x's type.
    @staticmethod
    def forward(ctx, x, weight, layer):
        y, slot = layer._forward(x.to(torch.bfloat16).contiguous(), weight.to(torch.bfloat16).contiguous())
        ctx.layer, ctx.slot = layer, slot
        return y

    @staticmethod
    def backward(ctx, dy):
        dx, dw = ctx.layer._backward(dy, ctx.slot)
        ctx.slot = None
        return dx, dw, None


class MetisLinear(torch.nn.Module):
    """``Y = X W`` with Metis W4A4G4 GeMMs in the forward and backward passes.

    Args:
        in_features, out_features: sizes (multiples of 256).
        k: rank of the spectral part of every operand (default ``default_rank``).
        s: oversampling of the randomized decomposition.
        sample_ratio: fraction of token rows sampled for the decomposition of X and dY
            (the weight is decomposed from all its rows).
        refresh_every: steps between randomized decompositions (the basis is reused in
            between and the factors recomputed every step).
        rounding: "sr" (stochastic) or "rn" (round to nearest) for the NVFP4 codes.
        seed: seed of the sampling, sketch and stochastic-rounding streams.
    """

    def __init__(self, in_features, out_features, k=None, s=8, sample_ratio=0.01, refresh_every=8,
                 rounding="sr", seed=0, device=None, dtype=torch.float32):
        super().__init__()
        if in_features % 256 or out_features % 256:
            raise ValueError("in_features and out_features must be multiples of 256")
        if rounding not in ("sr", "rn"):
            raise ValueError("rounding must be 'sr' or 'rn'")
        self.in_features, self.out_features = int(in_features), int(out_features)
        self.k = default_rank(in_features, out_features) if k is None else int(k)
        self.s, self.sample_ratio, self.refresh_every = int(s), float(sample_ratio), int(refresh_every)
        self.rounding = 1 if rounding == "sr" else 0
        self.seed = int(seed)
        self.weight = torch.nn.Parameter(torch.empty(in_features, out_features, device=device, dtype=dtype))
        bound = 1.0 / math.sqrt(in_features)
        with torch.no_grad():
            self.weight.uniform_(-bound, bound)
        self.step = 0
        self._bases = [_Basis(), _Basis(), _Basis()]   # X, W, dY

    # Checkpoint state beyond the weight: the step counter (it picks refresh steps and
    # enters the random streams) and the reused bases of X, W and dY, so that training
    # resumed from a checkpoint repeats the uninterrupted run bit for bit.
    def get_extra_state(self):
        return {"step": self.step,
                "bases": [None if b.V is None else (b.V.detach().cpu().clone(), b.shape) for b in self._bases]}

    def set_extra_state(self, state):
        self.step = int(state["step"])
        dev = self.weight.device
        for b, saved in zip(self._bases, state["bases"]):
            if saved is None:
                b.V, b.shape = None, None
            else:
                b.V, b.shape = saved[0].to(dev).clone(), tuple(saved[1])

    def extra_repr(self):
        return (f"in_features={self.in_features}, out_features={self.out_features}, k={self.k}, s={self.s}, "
                f"refresh_every={self.refresh_every}, rounding={'sr' if self.rounding else 'rn'}")

    def forward(self, x):
        if x.shape[-1] != self.in_features:
            raise ValueError(f"expected last dimension {self.in_features}, got {x.shape[-1]}")
        lead = x.shape[:-1]
        y = _MetisLinearFn.apply(x.reshape(-1, self.in_features), self.weight, self)
        return y.reshape(*lead, self.out_features)

    # -- one operand: basis bookkeeping, decomposition, residual quantization ----------
    def _l_k(self, rows, sampled):
        if not sampled:
            return rows
        return int(min(rows, max(math.ceil(self.sample_ratio * rows), self.k + self.s)))

    def _prepare(self, lib, M, op_id, step, sampled):
        rows, cols = M.shape
        basis = self._bases[op_id]
        refresh = step % self.refresh_every == 0 or basis.shape != (rows, cols)
        o = _Operand(rows, cols, self.k, M.device)
        if not refresh:
            o.factors.V.copy_(basis.V)
        lib.decompose(M, k=self.k, s=self.s, l_k=self._l_k(rows, sampled), seed=self.seed, operand_id=op_id,
                      refresh=refresh, step=step, factors=o.factors, rounding=self.rounding)
        if basis.shape != (rows, cols):
            basis.V, basis.shape = torch.empty_like(o.factors.V), (rows, cols)
        basis.V.copy_(o.factors.V)
        # tensor_scale 0: the decode scale g is chosen on the device from the operand's
        # magnitude, so gradients (about 1e-7 and below) keep their E4M3 block scales
        lib.residual_quantize_nvfp4(M, o.factors, rowwise=o.row, colwise=o.col, rounding=self.rounding,
                                    seed=self.seed, operand_id=op_id, step=step, tensor_scale=0.0)
        return o

    def _check_rows(self, rows):
        if rows % 256:
            raise ValueError(f"the number of tokens ({rows}) must be a multiple of 256")

    def _forward(self, x, w):
        self._check_rows(x.shape[0])
        lib, lock = _shared_context(x.device)
        step = self.step
        self.step += 1
        with lock:
            ox = self._prepare(lib, x, 0, step, sampled=True)
            ow = self._prepare(lib, w, 1, step, sampled=False)
            y = torch.empty(x.shape[0], self.out_features, dtype=torch.bfloat16, device=x.device)
            lib.linear_fwd(ox.struct, ow.struct, y)
        return y, (ox, ow, step)

    def _backward(self, dy, slot):
        ox, ow, step = slot
        dy = dy.to(torch.bfloat16).contiguous()
        lib, lock = _shared_context(dy.device)
        with lock:
            od = self._prepare(lib, dy, 2, step, sampled=True)
            dx = torch.empty(dy.shape[0], self.in_features, dtype=torch.bfloat16, device=dy.device)
            dw = torch.empty(self.in_features, self.out_features, dtype=torch.float32, device=dy.device)
            lib.linear_bwd(ox.struct, ow.struct, od.struct, dx, dw)
        return dx, dw
