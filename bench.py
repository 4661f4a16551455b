"""Benchmark of the Metis W4A4G4 linear layer (fwd + dX + dW) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config llama3_8b_mlp_up] [--no-cpu-baseline]

One step is the whole hot path on one batch: the randomized decomposition of
X, W and D (refreshed every 8 steps, reused otherwise), the residual NVFP4
quantization of each in both orientations, and the three fused GeMMs.  Every
step trains on a new token batch (X, D) -- the bench cycles through
``--batches`` distinct seeded draws that share the layer's outlier channels --
so the reused basis meets new data each step, as in training.  The
metric is effective TFLOP/s = 6 l m n / step time (useful GeMM flops only).

Workload: LLaMA-3 8B MLP up-projection at 8192 tokens (X 8192 x 4096,
W 4096 x 14336, D 8192 x 14336, k = 64, s = 8, l_k = 82, stochastic rounding),
synthetic anisotropic bf16 inputs.  The inputs (419 MB) exceed the 126 MB L2.

With N > 1 (launched by torch.distributed.run) every rank runs its own batch
of X and D with the shared W: weak scaling, no collective in the data path;
the time is the maximum over ranks.

``--impl reference`` times the CPU oracle on a bounded row sample of the same
workload (rank 0 only).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

NVFP4_OVER_BF16 = 9.0 / 2.25      # nominal dense tensor-core throughput ratio
DEFAULT_CONFIG = "llama3_8b_mlp_up"
METRIC = "effective TFLOP/s of Metis W4A4G4 linear fwd+bwd; % of NVFP4 MMA peak"
# DRAM bytes (read + write) of one launch of the fused GeMM (CTA-pair kernel) at the
# forward shape (8192 x 14336 x 4096, fold 256, bf16 out), from one ncu capture of this
# kernel version (bench.py --stage gemm; the summary sits under profiles/).
# Must be retaken whenever the kernel changes.
GEMM_FWD_DRAM_BYTES = 69.213184e6 + 193.452544e6
# DRAM bytes (read + write) of one launch of the residual quantizer on the benchmark's D
# (8192 x 14336, k = 64, SR), from one ncu capture of this kernel version
# (bench.py --stage resquant; the summary sits under profiles/). Must be retaken whenever the kernel changes.
RESQUANT_D_DRAM_BYTES = 248.5248e6 + 107.178752e6
RESQUANT_TRAFFIC_BASIS = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch on D (8192 x 14336), "
                          "bytes; the timed launches cover X, W and D")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this GPU while the timed region runs.

    Reads only.  With NVML (pynvml) a thread polls every ``period`` seconds and
    ``stop(t0, t1)`` keeps the samples taken between the host times t0 (just before the
    timed launches are issued) and t1 (after the closing synchronize), so the record covers
    the timed region itself even when it lasts a few tens of milliseconds.  Without NVML it
    falls back to ``nvidia-smi -lms 200`` over the same window (fewer samples)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"))

    def __init__(self, device, period=0.002, nvml=None):
        self.period = period
        self.samples = []          # (host time, sm MHz, max sm MHz, set of reason names)
        self.proc = None
        self.thread = None
        self.running = False
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.ident = str(getattr(device, "index", 0))
        self.nvml, self.handle = None, None
        try:
            if nvml is None:
                import pynvml as nvml
            nvml.nvmlInit()
            self.handle = nvml.nvmlDeviceGetHandleByUUID(self.ident)
            self.nvml = nvml
            self._sample_nvml()          # every query the poll makes works here, or NVML is not used
            self.samples.clear()
        except Exception:
            self.nvml = None

    def _reason_bits(self):
        nv = self.nvml
        out = []
        for name, suffix in self.REASONS:
            bit = getattr(nv, "nvmlClocksEventReason" + suffix, None)
            if bit is None:
                bit = getattr(nv, "nvmlClocksThrottleReason" + suffix)
            out.append((name, bit))
        return out

    def _sample_nvml(self):
        nv, h = self.nvml, self.handle
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        t = time.perf_counter()
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        active = reasons_fn(h)
        self.samples.append((t, float(sm), float(smax), {name for name, bit in self._reason_bits() if active & bit}))

    def _poll_nvml(self):
        while self.running:
            try:
                self._sample_nvml()
            except Exception:
                return
            time.sleep(self.period)

    def _read_smi(self):
        names = [name for name, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((time.perf_counter(), sm, smax,
                                 {nm for nm, val in zip(names, parts[5:9]) if val.lower() == "active"}))

    def start(self):
        self.running = True
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.ident}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t0=None, t1=None):
        self.running = False
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.nvml is None and self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no NVML and no nvidia-smi"], "samples": 0}
        inside = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        window = "timed region"
        if not inside:                       # nothing landed inside: report the nearest samples
            inside, window = self.samples, "around the timed region"
        sm = [x[1] for x in inside]
        reasons = set().union(*[x[3] for x in inside]) if inside else set()
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": inside[-1][2] if inside else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": ("nvml, every %.0f ms" % (1e3 * self.period)) if self.nvml else "nvidia-smi, every 200 ms",
                "window": window}


# ------------------------------------------------------------------ our arm
class Layer:
    """Device state of one Metis linear layer and its step.

    ``batches`` is a list of (X, D) device tensors; step t trains on batch
    t mod len(batches) with the one weight W, so each step brings new tokens.

    The three operands are independent until the GeMMs, so each is decomposed and
    quantized by its own libmetis context on its own CUDA stream (the single-CTA
    dense solves of X, W and D then overlap each other and the other operands'
    bandwidth-bound kernels); the GeMMs run on the caller's stream after joining
    the operand streams through events."""

    NAMES = ("X", "W", "D")

    def __init__(self, lib, ctx, cfg, batches, W, plain=False):
        self.lib, self.ctx, self.cfg = lib, ctx, cfg
        self.plain = plain   # plain NVFP4 (no decomposition, no fold): the baseline Metis improves on
        self.rounding = 1 if cfg["rounding"] == "sr" else 0
        self.batches = batches
        X, D = batches[0]
        self.mats = {"X": X, "W": W, "D": D}
        dev = W.device
        # X and W gate the forward GeMM, D only the backward; X's chain finishes last of the
        # two.  Stream priorities X > W > D > the GeMM stream, so when the three chains
        # overlap, free SMs go first to the chain that gates the forward GeMM longest.
        prio = {"X": -3, "W": -2, "D": -1}
        self.streams = {name: torch.cuda.Stream(dev, priority=prio[name]) for name in self.NAMES}
        self.ctxs = {}
        for name in self.NAMES:
            with torch.cuda.stream(self.streams[name]):
                self.ctxs[name] = lib.Context(dev.index)
        k, s = cfg["k"], cfg["s"]
        self.l_k = {"X": cfg["l_k"], "W": cfg["m"], "D": cfg["l_k"]}
        self.ops = {}
        for name, M in self.mats.items():
            rows, cols = M.shape
            f = None if plain else ctx.new_factors(rows, cols, k, s)
            row, col = ctx.new_nvfp4(rows, cols), ctx.new_nvfp4(cols, rows)
            self.ops[name] = (f, row, col, ctx.operand(row, col, f))
        l, m, n = cfg["l"], cfg["m"], cfg["n"]
        # activations and input gradients in bf16, the weight gradient in fp32 (the
        # boundary's output types; the GeMMs accumulate in fp32 either way)
        self.Y = torch.empty(l, n, dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty(l, m, dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty(m, n, dtype=torch.float32, device=dev)

    def profile(self, on):
        """CUDA events around the instrumented launches of every context (or off)."""
        self.ctx.profile_enable(on)
        for c in self.ctxs.values():
            c.profile_enable(on)

    def profile_read(self, kind):
        """(ms, launches, work) of one instrumented kernel kind over all contexts."""
        tot = [0.0, 0, 0.0]
        for c in [self.ctx] + list(self.ctxs.values()):
            ms, n, w = c.profile_read(kind)
            tot[0] += ms
            tot[1] += n
            tot[2] += w
        return tuple(tot)

    def step(self, t, operands=None, outputs=None):
        """One training step on batch t mod len(batches), or on explicit device operands
        (X, W, D) and outputs (Y, dX, dW) (the end-to-end run's double buffers; W must keep
        the shape of the layer's weight)."""
        cfg = self.cfg
        refresh = t % cfg["refresh_every"] == 0
        if operands is None:
            self.mats["X"], self.mats["D"] = self.batches[t % len(self.batches)]
        else:
            self.mats["X"], self.mats["W"], self.mats["D"] = operands
        if outputs is not None:
            self.Y, self.dX, self.dW = outputs
        main = torch.cuda.current_stream(self.Y.device)
        start = torch.cuda.Event()
        start.record(main)               # inputs in place, previous GeMMs issued
        ready = {}
        for i, name in enumerate(self.NAMES):
            stream = self.streams[name]
            stream.wait_event(start)
            with torch.cuda.stream(stream):
                ctx = self.ctxs[name]
                f, row, col, _ = self.ops[name]
                M = self.mats[name]
                if not self.plain:
                    ctx.decompose(M, k=cfg["k"], s=cfg["s"], l_k=self.l_k[name], seed=cfg["seed"], operand_id=i,
                                  refresh=refresh, step=t, factors=f, rounding=self.rounding)
                ctx.residual_quantize_nvfp4(M, f, row, col, rounding=self.rounding, seed=cfg["seed"],
                                            operand_id=i, step=t)
                ready[name] = torch.cuda.Event()
                ready[name].record(stream)
        main.wait_event(ready["X"])
        main.wait_event(ready["W"])
        self.ctx.linear_fwd(self.ops["X"][3], self.ops["W"][3], self.Y)
        main.wait_event(ready["D"])
        self.ctx.linear_bwd(self.ops["X"][3], self.ops["W"][3], self.ops["D"][3], self.dX, self.dW)

    def poll_device_status(self):
        st = self.ctx.poll_device_status()
        for c in self.ctxs.values():
            st |= c.poll_device_status()
        return st


class LoraStep:
    """One training step of the LoRA-SVD projection W = W_res + beta L2 L1 ("Full-Stack
    FP4", section 2.1) on the same batches: X, bf16(W_res) and D quantized to plain NVFP4
    (both orientations) on three streams; then the forward and input-gradient products
    with the bf16 branch in the FP4 GeMM's fold, the NVFP4 residual gradient, the two
    branch gradients on the caller's stream; the Cholesky-QR constraint on a stream of
    its own once the input-gradient product has read L2 and L1, so that it overlaps the
    residual gradient, the branch gradients and the next step's quantization (none of
    which read L2 or L1); the next forward product waits for it."""

    NAMES = ("X", "W", "D")

    def __init__(self, lib, ctx, cfg, batches, W):
        self.lib, self.ctx, self.cfg, self.batches = lib, ctx, cfg, batches
        dev = W.device
        l, m, n, k = cfg["l"], cfg["m"], cfg["n"], cfg["k"]
        self.k, self.beta = k, 1.0
        gen = torch.Generator(device=dev).manual_seed(cfg["seed"] + 17)
        self.L2 = torch.linalg.qr(torch.randn(m, k, device=dev, generator=gen))[0].contiguous()
        self.L1 = (0.05 * torch.randn(k, n, device=dev, generator=gen)).contiguous()
        self.mats = {"X": batches[0][0], "W": W, "D": batches[0][1]}
        self.streams = {name: torch.cuda.Stream(dev) for name in self.NAMES}
        self.ctxs = {}
        for name in self.NAMES:
            with torch.cuda.stream(self.streams[name]):
                self.ctxs[name] = lib.Context(dev.index)
        self.cstream = torch.cuda.Stream(dev)
        with torch.cuda.stream(self.cstream):
            self.cctx = lib.Context(dev.index)
        self.c_done = None
        self.q = {name: (ctx.new_nvfp4(*M.shape), ctx.new_nvfp4(M.shape[1], M.shape[0]))
                  for name, M in self.mats.items()}
        self.Y = torch.empty(l, n, dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty(l, m, dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty(m, n, dtype=torch.float32, device=dev)
        self.Tx = torch.empty(l, k, dtype=torch.float32, device=dev)
        self.Td = torch.empty(l, k, dtype=torch.float32, device=dev)
        self.dL2 = torch.empty(m, k, dtype=torch.float32, device=dev)
        self.dL1 = torch.empty(k, n, dtype=torch.float32, device=dev)

    def step(self, t):
        cfg, ctx = self.cfg, self.ctx
        self.mats["X"], self.mats["D"] = self.batches[t % len(self.batches)]
        main = torch.cuda.current_stream(self.Y.device)
        start = torch.cuda.Event()
        start.record(main)
        ready = {}
        for i, name in enumerate(self.NAMES):
            stream = self.streams[name]
            stream.wait_event(start)
            with torch.cuda.stream(stream):
                row, col = self.q[name]
                self.ctxs[name].residual_quantize_nvfp4(self.mats[name], None, row, col,
                                                        rounding=1 if name == "D" else 0, seed=cfg["seed"],
                                                        operand_id=i, step=t, tensor_scale=0.0)
                ready[name] = torch.cuda.Event()
                ready[name].record(stream)
        (xr, xc), (wr, wc), (dr, dc) = self.q["X"], self.q["W"], self.q["D"]
        X, D = self.mats["X"], self.mats["D"]
        main.wait_event(ready["X"])
        main.wait_event(ready["W"])
        self.finish()
        ctx.lora_linear(0, xr, wc, X, self.L2, self.L1, self.beta, self.Y, T=self.Tx)
        main.wait_event(ready["D"])
        ctx.lora_linear(1, dr, wr, D, self.L2, self.L1, self.beta, self.dX, T=self.Td)
        read = torch.cuda.Event()
        read.record(main)
        ctx.gemm_nvfp4(xc, dc, cfg["n"], self.dW)
        ctx.lora_branch_grad(X, self.Td, self.beta, self.dL2)
        ctx.lora_branch_grad(D, self.Tx, self.beta, self.dL1, transpose_out=True)
        self.cstream.wait_event(read)
        with torch.cuda.stream(self.cstream):
            self.cctx.lora_constrain(self.L2, self.L1)
            self.c_done = torch.cuda.Event()
            self.c_done.record(self.cstream)

    def finish(self):
        """The caller's stream waits for the last step's constraint."""
        if self.c_done is not None:
            torch.cuda.current_stream(self.Y.device).wait_event(self.c_done)

    def poll_device_status(self):
        st = self.ctx.poll_device_status() | self.cctx.poll_device_status()
        for c in self.ctxs.values():
            st |= c.poll_device_status()
        return st


def max_over_ranks(value, world, device):
    """The largest value over all ranks (a time measured on each rank's device)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_config(cfg, rank):
    """Weak scaling: every rank trains on its own tokens (X, D) with the shared W."""
    return dict(cfg, seed=cfg["seed"] + 1000 * rank)


def gen_operands(cfg, batches, rank=0):
    """W and `batches` token batches (X, D) of a configuration, pinned host bf16, generated
    on host threads (the seeded recipe of workloads/synth.py)."""
    from concurrent.futures import ThreadPoolExecutor
    rcfg = rank_config(cfg, rank)
    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        fw = ex.submit(synth.operand_matrix, cfg, "W")
        fb = [(ex.submit(synth.batch_matrix, rcfg, "X", b), ex.submit(synth.batch_matrix, rcfg, "D", b))
              for b in range(batches)]
        W = fw.result().pin_memory()
        host_batches = [(x.result().pin_memory(), d.result().pin_memory()) for x, d in fb]
    return W, host_batches


def timed_steps(layer, device, first, steps, world, barrier, per_step=False):
    """Time `steps` consecutive layer steps t = first .. (CUDA events on the caller's stream,
    synchronize and barrier on both sides); returns (total ms, per-step ms or None)."""
    stream = torch.cuda.current_stream(device)
    barrier()
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)] if per_step else None
    ev0.record(stream)
    for i, t in enumerate(range(first, first + steps)):
        if per_step:
            step_ev[i].record(stream)     # a step's operand work starts after the previous step's GeMMs
        layer.step(t)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    ms = ev0.elapsed_time(ev1)
    if not per_step:
        return ms, None
    bounds = step_ev + [ev1]
    return ms, [bounds[i].elapsed_time(bounds[i + 1]) for i in range(steps)]


def refresh_share(step_ms, first, refresh_every):
    """(refresh step ms, reuse step ms, amortised share) from per-step times."""
    refresh = [d for i, d in enumerate(step_ms) if (first + i) % refresh_every == 0]
    reuse = [d for i, d in enumerate(step_ms) if (first + i) % refresh_every != 0]
    if not refresh or not reuse:
        return (statistics.mean(refresh) if refresh else None), (statistics.median(reuse) if reuse else None), None
    r, n = statistics.mean(refresh), statistics.median(reuse)
    return r, n, (r - n) / (refresh_every * n)


def kernel_roofline(ms, n, work, peak, unit, bound, kernel, basis, traffic=None, traffic_basis=None):
    """One kernel's roofline entry from its CUDA-event-timed launches (work in flops or bytes)."""
    if not n or ms <= 0:
        return {"kernel": kernel, "bound": bound, "achieved": None, "peak": round(peak, 1), "unit": unit,
                "frac": None, "traffic": traffic, "launches_timed": 0}
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    achieved = work / (ms * 1e-3) / scale
    return {"kernel": kernel, "bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_basis": traffic_basis,
            "launches_timed": n, "us_per_launch": round(1e3 * ms / n, 2),
            "work_per_launch": round(work / n), "peak_basis": basis}


def run_e2e(layer, host_W, host_batches, device, first, steps, world, barrier):
    """End to end through the public API with host buffers: every step uploads its inputs (W,
    X, D) from pinned host memory and downloads its results (Y, dX, dW) into pinned host
    memory.  Copies run on two copy streams against double-buffered device operands and
    outputs, so step t+1's upload and step t's download overlap step t's compute."""
    h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    main = torch.cuda.current_stream(device)
    dev_in = [tuple(torch.empty_like(x, device=device) for x in (host_batches[0][0], host_W, host_batches[0][1]))
              for _ in range(2)]
    dev_out = [tuple(torch.empty_like(y) for y in (layer.Y, layer.dX, layer.dW)) for _ in range(2)]
    host_out = [tuple(torch.empty_like(y, device="cpu").pin_memory() for y in (layer.Y, layer.dX, layer.dW))
                for _ in range(2)]
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def upload(t):
        b = t % 2
        x, d = host_batches[t % len(host_batches)]
        h2d.wait_event(computed[b])            # the step two back has finished reading this buffer
        with torch.cuda.stream(h2d):
            for dst, src in zip(dev_in[b], (x, host_W, d)):
                dst.copy_(src, non_blocking=True)
            in_ready[b].record(h2d)

    saved = (layer.mats["X"], layer.mats["W"], layer.mats["D"], layer.Y, layer.dX, layer.dW)
    barrier()
    torch.cuda.synchronize(device)
    for b in range(2):                          # nothing to wait for yet
        computed[b].record(main)
        out_done[b].record(main)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    h2d.wait_event(computed[0])
    upload(first)
    for i, t in enumerate(range(first, first + steps)):
        b = t % 2
        main.wait_event(in_ready[b])
        main.wait_event(out_done[b])            # the download two steps back has read these outputs
        layer.step(t, operands=dev_in[b], outputs=dev_out[b])
        computed[b].record(main)
        if i + 1 < steps:
            upload(t + 1)
        d2h.wait_event(computed[b])
        with torch.cuda.stream(d2h):
            for dst, src in zip(host_out[b], dev_out[b]):
                dst.copy_(src, non_blocking=True)
            out_done[b].record(d2h)
    main.wait_event(out_done[(first + steps - 1) % 2])
    main.wait_event(out_done[(first + steps - 2) % 2])
    e1.record(main)
    torch.cuda.synchronize(device)
    barrier()
    layer.mats["X"], layer.mats["W"], layer.mats["D"], layer.Y, layer.dX, layer.dW = saved
    h2d_bytes = sum(v.numel() * v.element_size() for v in (host_W,) + host_batches[0])
    d2h_bytes = sum(v.numel() * v.element_size() for v in host_out[0])
    return e0.elapsed_time(e1), h2d_bytes, d2h_bytes


def config_line(lib, cfg_name, device, steps=8, warmup=3, batches=2, world=1, barrier=lambda: None):
    """A short run of another workload: effective TFLOP/s, ms per step, the main GeMM's
    fraction of the NVFP4 peak and the refresh share."""
    if cfg_name == "long_token_stress_r8":     # the stress workload again, refreshed every 8th step
        cfg = dict(synth.CONFIGS["long_token_stress"], refresh_every=8)
    else:
        cfg = synth.CONFIGS[cfg_name]
    host_W, host_batches = gen_operands(cfg, batches)
    W = host_W.to(device)
    dev_batches = [(x.to(device), d.to(device)) for x, d in host_batches]
    ctx = lib.Context(device.index)
    layer = Layer(lib, ctx, cfg, dev_batches, W)
    for t in range(warmup):
        layer.step(t)
    layer.profile(True)
    ms, step_ms = timed_steps(layer, device, warmup, steps, world, barrier, per_step=True)
    gemm = layer.profile_read(lib.PROF_GEMM)
    layer.profile(False)
    status = layer.poll_device_status()
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    flops = (2.0 if cfg["fwd_only"] else 6.0) * l * m * n
    r_ms, n_ms, share = refresh_share(step_ms, warmup, cfg["refresh_every"])
    out = {"workload": f"{cfg_name}: X {l}x{m}, W {m}x{n}, D {l}x{n}, k={cfg['k']}, s={cfg['s']}, "
                       f"l_k={cfg['l_k']}, refresh every {cfg['refresh_every']}",
           "value": round(flops / (ms / steps * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
           "ms_per_step": round(ms / steps, 4), "steps": steps, "warmup": warmup, "batches": batches,
           "gemm_tflops": round(gemm[2] / (gemm[0] * 1e-3) / 1e12, 1) if gemm[1] else None,
           "refresh_step_ms": None if r_ms is None else round(r_ms, 4),
           "reuse_step_ms": None if n_ms is None else round(n_ms, 4),
           "amortised_share": None if share is None else round(share, 4), "device_status": status}
    del layer, dev_batches, W
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, device):
    import spectral_quantized_gemm_b200 as lib
    cfg = synth.CONFIGS[args.config]
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    flops_per_step = 6.0 * l * m * n
    host_W, host_batches = gen_operands(cfg, args.batches, rank)
    dev_W = host_W.to(device)
    dev_batches = [(x.to(device), d.to(device)) for x, d in host_batches]
    ctx = lib.Context(device.index)
    layer = Layer(lib, ctx, cfg, dev_batches, dev_W)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for t in range(args.warmup):
        layer.step(t)
    torch.cuda.synchronize(device)
    status = layer.poll_device_status()
    if status:
        raise RuntimeError(f"device status bits {status} after warm-up")

    # ---- timed region: inputs resident in HBM
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.05)
    layer.profile(True)
    launches0 = lib.kernel_launches()
    t_region0 = time.perf_counter()
    ms, step_ms = timed_steps(layer, device, args.warmup, args.steps, world, barrier, per_step=True)
    t_region1 = time.perf_counter()
    launches = lib.kernel_launches() - launches0
    prof = {kind: layer.profile_read(kind) for kind in (lib.PROF_GEMM, lib.PROF_RESQUANT, lib.PROF_PROJECTION)}
    layer.profile(False)
    clk = clocks.stop(t_region0, t_region1)
    ms = max_over_ranks(ms, world, device)
    ms_per_step = ms / args.steps
    value = world * flops_per_step / (ms_per_step * 1e-3) / 1e12
    r_ms, n_ms, share = refresh_share(step_ms, args.warmup, cfg["refresh_every"])

    # ---- end to end through the public API: host inputs in, host results out, copies overlapped;
    # as many steps as the device-timed region (at least 4), so the pipeline's fill (the first
    # upload) and drain (the last download) weigh as little as the run length allows
    e2e_steps = max(4, args.steps)
    first = args.warmup + args.steps
    e2e_ms, h2d, d2h = run_e2e(layer, host_W, host_batches, device, first, e2e_steps, world, barrier)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_value = world * flops_per_step / (e2e_ms / e2e_steps * 1e-3) / 1e12
    status = layer.poll_device_status()

    # ---- plain NVFP4 on the same batches (no decomposition, no rank fold), same timing
    plain = Layer(lib, ctx, cfg, dev_batches, dev_W, plain=True)
    for t in range(3):
        plain.step(t)
    plain_ms, _ = timed_steps(plain, device, 3, args.steps, world, barrier)
    plain_ms = max_over_ranks(plain_ms / args.steps, world, device)
    status |= plain.poll_device_status()

    # ---- the LoRA-SVD projection's training step on the same batches, same timing
    lora = LoraStep(lib, ctx, cfg, dev_batches, dev_W)
    for t in range(3):
        lora.step(t)
    barrier()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q0.record(stream)
    for t in range(3, 3 + args.steps):
        lora.step(t)
    lora.finish()
    q1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    lora_ms = max_over_ranks(q0.elapsed_time(q1) / args.steps, world, device)
    status |= lora.poll_device_status()
    del lora, plain

    # the achievable FP4 MMA rate on this GPU (no memory traffic), beside the roofline
    mma_peak = ctx.nvfp4_mma_peak(iters=4096, reps=5)
    status |= ctx.poll_device_status()

    peaks, kind = measured_peaks()
    # the timed region lasts tens of milliseconds at full clock: the burst peaks apply
    nvfp4_peak = peaks["bf16_tflops"] * NVFP4_OVER_BF16
    nvfp4_sustained = peaks["bf16_tflops_sustained"] * NVFP4_OVER_BF16
    hbm = peaks["hbm_gbs"]
    gemm = kernel_roofline(*prof[lib.PROF_GEMM], nvfp4_peak, "TFLOP/s", "tensor",
                           "gemm_nvfp4_pair_kernel (fused FP4 GeMM + rank fold, CTA pairs; fwd, dX, dW)",
                           f"{kind} bf16 burst x {NVFP4_OVER_BF16:.0f} (nominal NVFP4/bf16 ratio)",
                           traffic=round(GEMM_FWD_DRAM_BYTES),
                           traffic_basis="ncu dram__bytes_read.sum + dram__bytes_write.sum of one forward-shape "
                                         "launch (bytes)")
    if gemm["achieved"] is not None:
        gemm["frac_of_sustained_peak"] = round(gemm["achieved"] / nvfp4_sustained, 4)
        gemm["frac_of_mma_microbenchmark"] = round(gemm["achieved"] / mma_peak, 4)
        gemm["frac_of_datasheet_9pf"] = round(gemm["achieved"] / 9000.0, 4)
    resq = kernel_roofline(*prof[lib.PROF_RESQUANT], hbm, "GB/s", "hbm",
                           "resquant_kernel (residual + NVFP4, both orientations; X, W, D)",
                           f"{kind} HBM copy bandwidth", traffic=RESQUANT_D_DRAM_BYTES,
                           traffic_basis=RESQUANT_TRAFFIC_BASIS)
    proj = kernel_roofline(*prof[lib.PROF_PROJECTION], hbm, "GB/s", "hbm",
                           "per-step projection P = M V (bf16 hi/lo tensor-core GeMM with its split and "
                           "reduction launches; X, W, D)", f"{kind} HBM copy bandwidth")
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 scales; fp32 accumulate)",
        "data": f"synthetic anisotropic bf16 (spikes on 2% of hidden dims + N(0,1) bulk), seeded; "
                f"{args.batches} token batches of X and D cycled (new tokens every step), one W",
        "config": {"workload": f"{args.config}: X {l}x{m}, W {m}x{n}, D {l}x{n}, k={cfg['k']}, s={cfg['s']}, "
                               f"l_k={cfg['l_k']}, refresh every {cfg['refresh_every']}, {cfg['rounding']} rounding",
                   "tokens_per_gpu": l, "parallelism": f"replicas x{world} (independent batches, shared W)",
                   "l2": "each step's inputs (419 MB) larger than the 126 MB L2; no flush",
                   "batches": args.batches,
                   "streams": "X, W and D decomposed and quantized on three streams; the GeMMs on one",
                   "outputs": "Y and dX bf16, dW fp32 (fp32 accumulation)",
                   "pct_of_nvfp4_peak": round(100 * value / (world * nvfp4_peak), 2),
                   "nvfp4_peak_tflops": round(nvfp4_peak, 1),
                   "nvfp4_peak_basis": f"bf16_tflops (burst) x {NVFP4_OVER_BF16:.0f} ({kind})"},
        "roofline": gemm,
        "rooflines": {"resquant": resq, "projection": proj},
        "nvfp4_mma_peak": {
            "value": round(mma_peak, 1), "unit": "TFLOP/s",
            "what": "tcgen05 kind::mxf4nvf4 block16 MMAs (CTA pairs, M=256 N=256 K=64) on resident "
                    "operands, no memory traffic: the rate the fused GeMM could reach"},
        "plain_nvfp4": {
            "value": round(world * flops_per_step / (plain_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(plain_ms, 4),
            "metis_over_plain": round(ms_per_step / plain_ms, 4),
            "what": "the same step with k = 0: residual = operand, plain NVFP4 in both orientations, "
                    "three FP4 GeMMs without the rank fold"},
        "lora_svd": {
            "value": round(world * flops_per_step / (lora_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(lora_ms, 4), "k": cfg["k"],
            "what": "LoRA-SVD projection (W = W_res + beta L2 L1, rank-k bf16 branch, NVFP4 residual) on the "
                    "same batches: plain NVFP4 quantization of X, bf16(W_res), D; forward and dX with the "
                    "branch in the FP4 GeMM fold; NVFP4 dW_res; branch gradients dL2, dL1; the Cholesky-QR "
                    "constraint (on its own stream, overlapping the gradients and the next quantization)"},
        "decomposition": {
            "refresh_every": cfg["refresh_every"],
            "refresh_steps_timed": sum(1 for i in range(args.steps) if (args.warmup + i) % cfg["refresh_every"] == 0),
            "refresh_step_ms": None if r_ms is None else round(r_ms, 4),
            "reuse_step_ms": None if n_ms is None else round(n_ms, 4),
            "amortised_share": None if share is None else round(share, 4),
            "basis": "(refresh step - reuse step) / (refresh_every x reuse step), CUDA events per step"},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": round(e2e_ms / e2e_steps, 4),
                "copies": "pinned host memory; uploads and downloads on two copy streams, double-buffered "
                          "operands and outputs, overlapping the step's compute"},
        "gpu_launches": launches,
        "device_status": status,
    }
    del layer
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        result["configs"] = {}
        for name in ("gpt2_small_mlp_up", "llama3_8b_down_reuse", "long_token_stress", "long_token_stress_r8"):
            result["configs"][name] = config_line(lib, name, device)
    return result


# ------------------------------------------------------------------ oracle arm
def oracle_sample_step(cfg, sample, state, t):
    """The oracle's work for one step on a bounded sample (rows of X and D, full W)."""
    from oracle import metis
    rnd = cfg["rounding"]
    opx = metis.prepare_operand(sample["X"], state["X"], seed=cfg["seed"], operand_id=0, step=t, rounding=rnd)
    opw = metis.prepare_operand(sample["W"], state["W"], seed=cfg["seed"], operand_id=1, step=t, rounding=rnd)
    opd = metis.prepare_operand(sample["D"], state["D"], seed=cfg["seed"], operand_id=2, step=t, rounding=rnd)
    metis.linear_fwd(opx, opw)
    metis.linear_bwd(opx, opw, opd)


def oracle_setup(cfg, rows, cols):
    """Bounded sub-problem: the first `rows` token rows of X and D and the first
    `cols` output columns of W and D.  The three operands' bases are refreshed once here;
    the time that takes is returned, so that a step can carry 1 / refresh_every of it
    (the refresh the device step amortizes)."""
    from oracle import decompose
    full = {n: synth.operand_matrix(cfg, n, as_numpy=True) for n in ("X", "W", "D")}
    sample = {"X": full["X"][:rows], "W": np.ascontiguousarray(full["W"][:, :cols]),
              "D": np.ascontiguousarray(full["D"][:rows, :cols])}
    state = {}
    t0 = time.perf_counter()
    for i, n in enumerate(("X", "W", "D")):
        l_k = min(cfg["l_k"], rows) if n != "W" else sample[n].shape[0]
        state[n] = decompose.refresh_basis(sample[n], cfg["k"], cfg["s"], max(l_k, cfg["k"] + cfg["s"]),
                                           cfg["seed"], i, 0)["V"]
    return sample, state, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((d.get("num_threads", 1) for d in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def sample_text(cfg, rows, cols, dt, t_refresh):
    return (f"sub-problem of {rows}/{cfg['l']} token rows x {cols}/{cfg['n']} output columns "
            f"(X {rows}x{cfg['m']}, W {cfg['m']}x{cols}, D {rows}x{cols}): per-step factors, residual NVFP4 "
            f"in both orientations, fwd, dX, dW, plus 1/{cfg['refresh_every']} of the three bases' refresh "
            f"({t_refresh:.1f} s); {dt:.1f} s per step; value = 6*rows*m*cols / time")


def cpu_baseline(cfg, rows, cols, steps=1):
    sample, state, t_refresh = oracle_setup(cfg, rows, cols)
    t0 = time.perf_counter()
    for t in range(steps):
        oracle_sample_step(cfg, sample, state, t)
    dt = (time.perf_counter() - t0) / steps + t_refresh / cfg["refresh_every"]
    flops = 6.0 * rows * cfg["m"] * cols
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": sample_text(cfg, rows, cols, dt, t_refresh)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg = synth.CONFIGS[args.config]
    rows, cols = args.ref_rows, args.ref_cols
    sample, state, t_refresh = oracle_setup(cfg, rows, cols)
    for t in range(args.warmup):
        oracle_sample_step(cfg, sample, state, t)
    t0 = time.perf_counter()
    for t in range(args.warmup, args.warmup + args.steps):
        oracle_sample_step(cfg, sample, state, t)
    dt = (time.perf_counter() - t0) / args.steps + t_refresh / cfg["refresh_every"]
    flops = 6.0 * rows * cfg["m"] * cols
    value = flops / dt / 1e12
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    cb = {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
          "sample": sample_text(cfg, rows, cols, dt, t_refresh)}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic anisotropic bf16, seeded",
            "config": {"workload": f"{args.config}: X {l}x{m}, W {m}x{n}, D {l}x{n}, k={cfg['k']}",
                       "sample_rows": rows, "sample_cols": cols},
            "cpu_baseline": cb, "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def run_stage(args, device):
    """Profiling mode (``--stage``): issue one stage of the benchmark step ``--reps`` times on
    the benchmark workload's own operands and exit, for a profiler to capture by kernel
    name.  Prints no benchmark line and times nothing.

    resquant   the residual quantization of D (both orientations, rank-k factors)
    decompose  the per-step factor update of X (projection, eigensolve, factors)
    gemm       the forward fused GeMM of the layer (FP4 + rank fold, bf16 out)
    step       whole layer steps"""
    import spectral_quantized_gemm_b200 as lib
    cfg = synth.CONFIGS[args.config]
    W = synth.operand_matrix(cfg, "W").to(device)
    batches = [(synth.batch_matrix(cfg, "X", 0).to(device), synth.batch_matrix(cfg, "D", 0).to(device))]
    ctx = lib.Context(device.index)
    layer = Layer(lib, ctx, cfg, batches, W)
    layer.step(0)                         # refresh: the bases every stage starts from
    torch.cuda.synchronize(device)
    rnd = layer.rounding
    for t in range(1, args.reps + 1):
        if args.stage == "step":
            layer.step(t)
            continue
        name = {"resquant": "D", "decompose": "X", "gemm": "X"}[args.stage]
        f, row, col, _ = layer.ops[name]
        M = layer.mats[name]
        i = layer.NAMES.index(name)
        if args.stage == "resquant":
            ctx.residual_quantize_nvfp4(M, f, row, col, rounding=rnd, seed=cfg["seed"], operand_id=i, step=t)
        elif args.stage == "decompose":
            l_k = layer.l_k[name]
            ctx.decompose(M, k=cfg["k"], s=cfg["s"], l_k=l_k, seed=cfg["seed"], operand_id=i, refresh=False, step=t,
                          factors=f, rounding=rnd)
        else:
            ctx.linear_fwd(layer.ops["X"][3], layer.ops["W"][3], layer.Y)
    torch.cuda.synchronize(device)
    status = layer.poll_device_status()
    print(f"stage {args.stage}: {args.config}, {args.reps} repetitions, device status {status}", flush=True)
    return status


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=16)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the short runs of the other workloads")
    ap.add_argument("--batches", type=int, default=4, help="distinct token batches (X, D) cycled over the steps")
    ap.add_argument("--ref-rows", type=int, default=256, help="token rows of the oracle's bounded sample")
    ap.add_argument("--ref-cols", type=int, default=1024, help="output columns of the oracle's bounded sample")
    ap.add_argument("--stage", choices=["resquant", "decompose", "gemm", "step"],
                    help="profiling mode: run one stage --reps times for a profiler; no benchmark line")
    ap.add_argument("--reps", type=int, default=3, help="repetitions of --stage")
    args = ap.parse_args()
    if args.stage:
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        raise SystemExit(1 if run_stage(args, device) else 0)
    if args.warmup < 3:
        raise SystemExit("need at least 3 warm-up steps")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    res = run_ours(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(synth.CONFIGS[args.config], args.ref_rows, args.ref_cols)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
