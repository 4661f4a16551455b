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
# kernel version (profile_case.py gemm --bf16; the summary sits under profiles/).
# Must be retaken whenever the kernel changes.
GEMM_FWD_DRAM_BYTES = 69.383424e6 + 192.398336e6


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
        self.streams = {name: torch.cuda.Stream(dev) for name in self.NAMES}
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

    def step(self, t):
        cfg = self.cfg
        refresh = t % cfg["refresh_every"] == 0
        self.mats["X"], self.mats["D"] = self.batches[t % len(self.batches)]
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


def run_ours(args, rank, world, device):
    import spectral_quantized_gemm_b200 as lib
    cfg = synth.CONFIGS[args.config]
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    flops_per_step = 6.0 * l * m * n
    rcfg = rank_config(cfg, rank)
    host_W = synth.operand_matrix(cfg, "W").pin_memory()
    host_batches = [(synth.batch_matrix(rcfg, "X", b).pin_memory(), synth.batch_matrix(rcfg, "D", b).pin_memory())
                    for b in range(args.batches)]
    dev_W = host_W.to(device)
    dev_batches = [(x.to(device), d.to(device)) for x, d in host_batches]
    ctx = lib.Context(device.index)
    layer = Layer(lib, ctx, cfg, dev_batches, dev_W)
    stream = torch.cuda.current_stream(device)

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
    ctx.profile_enable(True)
    launches0 = lib.kernel_launches()
    barrier()
    torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_region0 = time.perf_counter()
    ev0.record(stream)
    for i, t in enumerate(range(args.warmup, args.warmup + args.steps)):
        step_ev[i].record(stream)     # a step's operand work starts after the previous step's GeMMs
        layer.step(t)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    t_region1 = time.perf_counter()
    barrier()
    bounds = step_ev + [ev1]
    step_ms = [bounds[i].elapsed_time(bounds[i + 1]) for i in range(args.steps)]
    refresh_ms = [d for i, d in enumerate(step_ms) if (args.warmup + i) % cfg["refresh_every"] == 0]
    normal_ms = [d for i, d in enumerate(step_ms) if (args.warmup + i) % cfg["refresh_every"] != 0]
    launches = lib.kernel_launches() - launches0
    gemm_ms, gemm_n, gemm_flops = ctx.profile_read()
    ctx.profile_enable(False)
    clk = clocks.stop(t_region0, t_region1)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world, device)
    ms_per_step = ms / args.steps
    value = world * flops_per_step / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the public API: host inputs in, host results out
    out_host = {"Y": torch.empty_like(layer.Y, device="cpu").pin_memory(),
                "dX": torch.empty_like(layer.dX, device="cpu").pin_memory(),
                "dW": torch.empty_like(layer.dW, device="cpu").pin_memory()}
    h2d = sum(v.numel() * v.element_size() for v in (host_W,) + host_batches[0])
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    e2e_steps = max(2, min(args.steps, 6))
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(args.warmup + args.steps, args.warmup + args.steps + e2e_steps):
        b = t % len(dev_batches)
        dev_W.copy_(host_W, non_blocking=True)
        dev_batches[b][0].copy_(host_batches[b][0], non_blocking=True)
        dev_batches[b][1].copy_(host_batches[b][1], non_blocking=True)
        layer.step(t)
        out_host["Y"].copy_(layer.Y, non_blocking=True)
        out_host["dX"].copy_(layer.dX, non_blocking=True)
        out_host["dW"].copy_(layer.dW, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_value = world * flops_per_step / (e2e_ms / e2e_steps * 1e-3) / 1e12
    status = layer.poll_device_status()

    # ---- plain NVFP4 on the same batches (no decomposition, no rank fold), same timing
    plain = Layer(lib, ctx, cfg, dev_batches, dev_W, plain=True)
    for t in range(3):
        plain.step(t)
    barrier()
    torch.cuda.synchronize(device)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for t in range(3, 3 + args.steps):
        plain.step(t)
    p1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    plain_ms = p0.elapsed_time(p1) / args.steps
    plain_ms = max_over_ranks(plain_ms, world, device)
    status |= plain.poll_device_status()

    # ---- the LoRA-SVD projection's training step on the same batches, same timing
    lora = LoraStep(lib, ctx, cfg, dev_batches, dev_W)
    for t in range(3):
        lora.step(t)
    barrier()
    torch.cuda.synchronize(device)
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

    # the achievable FP4 MMA rate on this GPU (no memory traffic), beside the roofline
    mma_peak = ctx.nvfp4_mma_peak(iters=4096, reps=5)
    status |= ctx.poll_device_status()

    peaks, kind = measured_peaks()
    peak = peaks["bf16_tflops_sustained"] * NVFP4_OVER_BF16
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
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
                   "pct_of_nvfp4_peak": round(100 * value / (world * peak), 2),
                   "nvfp4_peak_tflops": round(peak, 1),
                   "nvfp4_peak_basis": f"bf16_tflops_sustained x {NVFP4_OVER_BF16:.0f} ({kind})"},
        "roofline": {"bound": "tensor", "kernel": "gemm_nvfp4_pair_kernel (fused FP4 GeMM + fold, CTA pairs)",
                     "achieved": None if achieved is None else round(achieved, 1), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": None if achieved is None else round(achieved / peak, 4),
                     "traffic": round(GEMM_FWD_DRAM_BYTES),
                     "traffic_basis": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one forward-shape "
                                      "launch (bytes); the timed launches are the fwd, dX and dW GeMMs",
                     "launches_timed": gemm_n,
                     "peak_basis": f"{kind} bf16 sustained x {NVFP4_OVER_BF16:.0f} (nominal NVFP4/bf16 ratio)"},
        "nvfp4_mma_peak": {
            "value": round(mma_peak, 1), "unit": "TFLOP/s",
            "gemm_frac": None if achieved is None else round(achieved / mma_peak, 4),
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
            "refresh_steps_timed": len(refresh_ms),
            "refresh_step_ms": round(statistics.mean(refresh_ms), 4) if refresh_ms else None,
            "reuse_step_ms": round(statistics.median(normal_ms), 4) if normal_ms else None,
            "amortised_share": (round((statistics.mean(refresh_ms) - statistics.median(normal_ms))
                                      / (cfg["refresh_every"] * statistics.median(normal_ms)), 4)
                                if refresh_ms and normal_ms else None),
            "basis": "(refresh step - reuse step) / (refresh_every x reuse step), CUDA events per step"},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": launches,
        "device_status": status,
    }
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
    `cols` output columns of W and D (bases refreshed once, untimed)."""
    from oracle import decompose
    full = {n: synth.operand_matrix(cfg, n, as_numpy=True) for n in ("X", "W", "D")}
    sample = {"X": full["X"][:rows], "W": np.ascontiguousarray(full["W"][:, :cols]),
              "D": np.ascontiguousarray(full["D"][:rows, :cols])}
    state = {}
    for i, n in enumerate(("X", "W", "D")):
        l_k = min(cfg["l_k"], rows) if n != "W" else sample[n].shape[0]
        state[n] = decompose.refresh_basis(sample[n], cfg["k"], cfg["s"], max(l_k, cfg["k"] + cfg["s"]),
                                           cfg["seed"], i, 0)["V"]
    return sample, state


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((d.get("num_threads", 1) for d in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def sample_text(cfg, rows, cols, dt):
    return (f"sub-problem of {rows}/{cfg['l']} token rows x {cols}/{cfg['n']} output columns "
            f"(X {rows}x{cfg['m']}, W {cfg['m']}x{cols}, D {rows}x{cols}): per-step factors, residual NVFP4 "
            f"in both orientations, fwd, dX, dW; {dt:.1f} s per step; value = 6*rows*m*cols / time")


def cpu_baseline(cfg, rows, cols, steps=1):
    sample, state = oracle_setup(cfg, rows, cols)
    t0 = time.perf_counter()
    for t in range(steps):
        oracle_sample_step(cfg, sample, state, t)
    dt = (time.perf_counter() - t0) / steps
    flops = 6.0 * rows * cfg["m"] * cols
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": sample_text(cfg, rows, cols, dt)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg = synth.CONFIGS[args.config]
    rows, cols = args.ref_rows, args.ref_cols
    sample, state = oracle_setup(cfg, rows, cols)
    for t in range(args.warmup):
        oracle_sample_step(cfg, sample, state, t)
    t0 = time.perf_counter()
    for t in range(args.warmup, args.warmup + args.steps):
        oracle_sample_step(cfg, sample, state, t)
    dt = (time.perf_counter() - t0) / args.steps
    flops = 6.0 * rows * cfg["m"] * cols
    value = flops / dt / 1e12
    l, m, n = cfg["l"], cfg["m"], cfg["n"]
    cb = {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
          "sample": sample_text(cfg, rows, cols, dt)}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic anisotropic bf16, seeded",
            "config": {"workload": f"{args.config}: X {l}x{m}, W {m}x{n}, D {l}x{n}, k={cfg['k']}",
                       "sample_rows": rows, "sample_cols": cols},
            "cpu_baseline": cb, "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=16)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batches", type=int, default=4, help="distinct token batches (X, D) cycled over the steps")
    ap.add_argument("--ref-rows", type=int, default=256, help="token rows of the oracle's bounded sample")
    ap.add_argument("--ref-cols", type=int, default=1024, help="output columns of the oracle's bounded sample")
    args = ap.parse_args()
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
