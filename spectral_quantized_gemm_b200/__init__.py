"""Python binding of libmetis, the B200 implementation of the Metis W4A4G4 linear layer.

Method: "Metis: Training LLMs with FP4 Quantization" (ICLR 2026; papernotes.org
notes).  Every call here marshals arguments into the C ABI declared in
``include/metis.h`` and runs on the GPU inside ``libmetis.so``; PyTorch only
provides device memory and the current CUDA stream.  There is no CPU path: if
the library is missing, importing this package fails.

Typical use (one operand):

    ctx = Context()
    st = ctx.new_factors(rows, cols, k)
    ctx.decompose(M, k=k, s=s, l_k=l_k, seed=0, operand_id=0, refresh=True, step=0, factors=st)
    row, col = ctx.new_nvfp4(rows, cols), ctx.new_nvfp4(cols, rows)
    ctx.residual_quantize_nvfp4(M, st, rowwise=row, colwise=col, rounding=1, seed=0, operand_id=0, step=0)
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmetis.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with `python spectral_quantized_gemm_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

c_i32, c_i64, c_u32, c_u64, c_f32, c_p = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64,
                                           ctypes.c_float, ctypes.c_void_p)

METIS_OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_ARCH", 5: "ERR_CUDA",
                6: "ERR_WORKSPACE"}
DEV_NUMERIC, DEV_NONFINITE, DEV_TIMEOUT = 1, 2, 4
OUT_F32, OUT_BF16 = 0, 1

EXPORTED = ["metis_create", "metis_destroy", "metis_set_stream", "metis_status_str", "metis_last_error",
            "metis_poll_device_status", "metis_nvfp4_codes_bytes", "metis_nvfp4_scales_bytes",
            "metis_decompose", "metis_residual_quantize_nvfp4", "metis_quantize_nvfp4_f32", "metis_gemm_nvfp4",
            "metis_linear_fwd", "metis_linear_bwd", "metis_kernel_launches", "metis_profile_enable",
            "metis_profile_read", "metis_residual_quantize_nvfp4_noalloc", "metis_dequantize_nvfp4",
            "metis_nvfp4_mma_peak", "metis_selftest_wait_timeout", "metis_lora_linear",
            "metis_lora_branch_grad", "metis_lora_constrain", "metis_lora_realign",
            "metis_residual_quantize_nvfp4_dump", "metis_profile_read_kind", "metis_set_sm_count_target",
            "metis_selftest_numeric"]

PROF_GEMM, PROF_RESQUANT, PROF_PROJECTION = 0, 1, 2


class Matrix(ctypes.Structure):
    _fields_ = [("data", c_p), ("rows", c_i64), ("cols", c_i64), ("ld", c_i64)]


class Nvfp4Struct(ctypes.Structure):
    _fields_ = [("codes", c_p), ("scales", c_p), ("tensor_scale", c_p), ("outer", c_i64), ("inner", c_i64)]


class FactorsStruct(ctypes.Structure):
    _fields_ = [("rows", c_i64), ("cols", c_i64), ("k", c_i32), ("V", c_p), ("U", c_p), ("S", c_p),
                ("Uq", Nvfp4Struct), ("Vq", Nvfp4Struct), ("sampled_rows", c_p), ("omega", c_p)]


class DecompParams(ctypes.Structure):
    _fields_ = [("k", c_i32), ("s", c_i32), ("l_k", c_i32), ("seed", c_u64), ("operand_id", c_u32),
                ("rounding", c_i32)]


class QuantParams(ctypes.Structure):
    _fields_ = [("rounding", c_i32), ("seed", c_u64), ("operand_id", c_u32), ("step", c_u32),
                ("tensor_scale", c_f32)]


class OperandStruct(ctypes.Structure):
    _fields_ = [("rowwise", ctypes.POINTER(Nvfp4Struct)), ("colwise", ctypes.POINTER(Nvfp4Struct)),
                ("f", ctypes.POINTER(FactorsStruct))]


def _sig(name, restype, *args):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(args)
    return fn


_create = _sig("metis_create", c_i32, ctypes.c_int, c_p, ctypes.POINTER(c_p))
_destroy = _sig("metis_destroy", None, c_p)
_set_stream = _sig("metis_set_stream", c_i32, c_p, c_p)
_set_sm_target = _sig("metis_set_sm_count_target", c_i32, c_p, ctypes.c_int)
_status_str = _sig("metis_status_str", ctypes.c_char_p, c_i32)
_last_error = _sig("metis_last_error", ctypes.c_char_p, c_p)
_poll = _sig("metis_poll_device_status", c_i32, c_p, ctypes.POINTER(c_u32), ctypes.c_int)
_codes_bytes = _sig("metis_nvfp4_codes_bytes", c_i64, c_i64, c_i64)
_scales_bytes = _sig("metis_nvfp4_scales_bytes", c_i64, c_i64, c_i64)
_decompose = _sig("metis_decompose", c_i32, c_p, ctypes.POINTER(Matrix), ctypes.POINTER(DecompParams),
                  ctypes.c_int, c_u32, ctypes.POINTER(FactorsStruct))
_resq = _sig("metis_residual_quantize_nvfp4", c_i32, c_p, ctypes.POINTER(Matrix), ctypes.POINTER(FactorsStruct),
             ctypes.POINTER(QuantParams), ctypes.POINTER(Nvfp4Struct), ctypes.POINTER(Nvfp4Struct))
_resq_noalloc = _sig("metis_residual_quantize_nvfp4_noalloc", c_i32, c_p, ctypes.POINTER(Matrix),
                     ctypes.POINTER(FactorsStruct), ctypes.POINTER(QuantParams), ctypes.POINTER(Nvfp4Struct),
                     ctypes.POINTER(Nvfp4Struct))
_resq_dump = _sig("metis_residual_quantize_nvfp4_dump", c_i32, c_p, ctypes.POINTER(Matrix),
                  ctypes.POINTER(FactorsStruct), ctypes.POINTER(QuantParams), ctypes.POINTER(Nvfp4Struct),
                  ctypes.POINTER(Nvfp4Struct), c_p, c_i64)
_dequant = _sig("metis_dequantize_nvfp4", c_i32, c_p, ctypes.POINTER(Nvfp4Struct), c_p, c_i64)
_mma_peak = _sig("metis_nvfp4_mma_peak", c_i32, c_p, c_i64, ctypes.POINTER(ctypes.c_double))
_wait_selftest = _sig("metis_selftest_wait_timeout", c_i32, c_p, c_i64)
_numeric_selftest = _sig("metis_selftest_numeric", c_i32, c_p)
_quant_f32 = _sig("metis_quantize_nvfp4_f32", c_i32, c_p, c_p, c_i64, c_i64, c_i64, ctypes.POINTER(QuantParams),
                  ctypes.POINTER(Nvfp4Struct), ctypes.POINTER(Nvfp4Struct))
_gemm = _sig("metis_gemm_nvfp4", c_i32, c_p, ctypes.POINTER(Nvfp4Struct), ctypes.POINTER(Nvfp4Struct), c_i64, c_p,
             c_p, c_i32, c_p, c_p, c_i64, c_i32)
_fwd = _sig("metis_linear_fwd", c_i32, c_p, ctypes.POINTER(OperandStruct), ctypes.POINTER(OperandStruct), c_p,
            c_i64, c_i32)
_bwd = _sig("metis_linear_bwd", c_i32, c_p, ctypes.POINTER(OperandStruct), ctypes.POINTER(OperandStruct),
            ctypes.POINTER(OperandStruct), c_p, c_i64, c_i32, c_p, c_i64)
_lora_linear = _sig("metis_lora_linear", c_i32, c_p, c_i32, ctypes.POINTER(Nvfp4Struct), ctypes.POINTER(Nvfp4Struct),
                    ctypes.POINTER(Matrix), c_p, c_p, c_i32, c_f32, c_p, c_p, c_i64, c_i32)
_lora_grad = _sig("metis_lora_branch_grad", c_i32, c_p, ctypes.POINTER(Matrix), c_p, c_i32, c_f32, c_i32, c_p)
_lora_constrain = _sig("metis_lora_constrain", c_i32, c_p, c_p, c_i64, c_p, c_i64, c_i32)
_lora_realign = _sig("metis_lora_realign", c_i32, c_p, c_p, c_i64, c_i64, c_i64, c_p, c_p, c_i32, c_f32,
                     ctypes.POINTER(DecompParams), c_u32, ctypes.POINTER(FactorsStruct), c_p)

_launches = _sig("metis_kernel_launches", c_u64)
_prof_enable = _sig("metis_profile_enable", c_i32, c_p, ctypes.c_int)
_prof_read = _sig("metis_profile_read", c_i32, c_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_i64),
                  ctypes.POINTER(ctypes.c_double))
_prof_read_kind = _sig("metis_profile_read_kind", c_i32, c_p, c_i32, ctypes.POINTER(ctypes.c_double),
                       ctypes.POINTER(c_i64), ctypes.POINTER(ctypes.c_double))


def kernel_launches():
    """Kernels launched by libmetis in this process so far."""
    return int(_launches())


class MetisError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def status_str(status):
    return _status_str(status).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class Nvfp4:
    """Device buffers of one NVFP4 tensor (outer x inner, blocks along inner)."""

    def __init__(self, outer, inner, device="cuda"):
        self.outer, self.inner = int(outer), int(inner)
        self.codes = torch.zeros(int(_codes_bytes(outer, inner)), dtype=torch.uint8, device=device)
        self.scales = torch.zeros(int(_scales_bytes(outer, inner)), dtype=torch.uint8, device=device)
        self.tensor_scale = torch.ones(4, dtype=torch.float32, device=device)
        self.struct = Nvfp4Struct(self.codes.data_ptr(), self.scales.data_ptr(), self.tensor_scale.data_ptr(),
                                  self.outer, self.inner)


class Factors:
    """Caller-owned factor state of one operand: V (basis), U, S and their NVFP4 copies."""

    def __init__(self, rows, cols, k, s=0, l_k=0, device="cuda", keep_sketch=False):
        self.rows, self.cols, self.k = int(rows), int(cols), int(k)
        self.V = torch.zeros(cols, k, dtype=torch.float32, device=device)
        self.U = torch.zeros(rows, k, dtype=torch.float32, device=device)
        self.S = torch.zeros(max(k, 1), dtype=torch.float32, device=device)
        self.Uq = Nvfp4(128, rows, device)
        self.Vq = Nvfp4(128, cols, device)
        self.sampled_rows = torch.zeros(max(l_k, 1), dtype=torch.int32, device=device) if keep_sketch else None
        self.omega = torch.zeros(cols, max(k + s, 1), dtype=torch.float32, device=device) if keep_sketch else None
        self.struct = FactorsStruct(self.rows, self.cols, self.k, self.V.data_ptr(), self.U.data_ptr(),
                                    self.S.data_ptr(), self.Uq.struct, self.Vq.struct,
                                    None if self.sampled_rows is None else self.sampled_rows.data_ptr(),
                                    None if self.omega is None else self.omega.data_ptr())


def _matrix(M):
    if M.dtype != torch.bfloat16 or M.dim() != 2 or M.stride(1) != 1:
        raise ValueError("expected a row-major 2-D bf16 CUDA tensor")
    return Matrix(M.data_ptr(), M.shape[0], M.shape[1], M.stride(0))


class Context:
    """A libmetis context bound to one device; work goes to torch's current stream."""

    def __init__(self, device=None):
        if not torch.cuda.is_available():
            raise RuntimeError("libmetis needs a CUDA device (sm_100)")
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        handle = c_p()
        st = _create(self.device.index, c_p(torch.cuda.current_stream(self.device).cuda_stream),
                     ctypes.byref(handle))
        if st != METIS_OK:
            raise MetisError(st, status_str(st))
        self._h = handle

    def close(self):
        if getattr(self, "_h", None):
            _destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _call(self, fn, *args):
        _set_stream(self._h, c_p(torch.cuda.current_stream(self.device).cuda_stream))
        st = fn(self._h, *args)
        if st != METIS_OK:
            raise MetisError(st, _last_error(self._h).decode())

    # -- allocation helpers ------------------------------------------------
    def new_nvfp4(self, outer, inner):
        return Nvfp4(outer, inner, self.device)

    def new_factors(self, rows, cols, k, s=0, l_k=0, keep_sketch=False):
        return Factors(rows, cols, k, s, l_k, self.device, keep_sketch)

    # -- the C ABI ---------------------------------------------------------
    def set_sm_count_target(self, n):
        """Size this context's later launches for n SMs (0: the device's count)."""
        st = _set_sm_target(self._h, int(n))
        if st != METIS_OK:
            raise MetisError(st, _last_error(self._h).decode())

    def poll_device_status(self, clear=True):
        bits = c_u32(0)
        self._call(_poll, ctypes.byref(bits), int(clear))
        return bits.value

    def decompose(self, M, k, s, l_k, seed, operand_id, refresh, step, factors, rounding=0):
        p = DecompParams(k, s, l_k, seed, operand_id, rounding)
        self._call(_decompose, ctypes.byref(_matrix(M)), ctypes.byref(p), int(bool(refresh)), step,
                   ctypes.byref(factors.struct))

    def residual_quantize_nvfp4(self, M, factors, rowwise=None, colwise=None, rounding=0, seed=0, operand_id=0,
                                step=0, tensor_scale=1.0):
        q = QuantParams(rounding, seed, operand_id, step, tensor_scale)
        self._call(_resq, ctypes.byref(_matrix(M)), None if factors is None else ctypes.byref(factors.struct),
                   ctypes.byref(q), None if rowwise is None else ctypes.byref(rowwise.struct),
                   None if colwise is None else ctypes.byref(colwise.struct))

    def residual_quantize_nvfp4_dump(self, M, factors, rowwise, colwise, residual, rounding=0, seed=0, operand_id=0,
                                     step=0, tensor_scale=1.0):
        """Both orientations, plus the fp32 residual the quantizer rounded (parity surface)."""
        if residual.dtype != torch.float32 or residual.dim() != 2 or residual.stride(1) != 1:
            raise ValueError("residual: expected a row-major 2-D fp32 CUDA tensor")
        q = QuantParams(rounding, seed, operand_id, step, tensor_scale)
        self._call(_resq_dump, ctypes.byref(_matrix(M)), None if factors is None else ctypes.byref(factors.struct),
                   ctypes.byref(q), ctypes.byref(rowwise.struct), ctypes.byref(colwise.struct), _ptr(residual),
                   residual.stride(0))

    def residual_quantize_nvfp4_noalloc(self, M, factors, rowwise, colwise, rounding=0, seed=0, operand_id=0,
                                        step=0, tensor_scale=1.0):
        """Allocation-free residual quantization: libmetis calls no cudaMalloc here
        (fixed 6 MiB device scratch; rows + cols <= 24576)."""
        q = QuantParams(rounding, seed, operand_id, step, tensor_scale)
        self._call(_resq_noalloc, ctypes.byref(_matrix(M)), None if factors is None else ctypes.byref(factors.struct),
                   ctypes.byref(q), ctypes.byref(rowwise.struct), ctypes.byref(colwise.struct))

    def quantize_nvfp4_f32(self, R, rowwise=None, colwise=None, rounding=0, seed=0, operand_id=0, step=0,
                           tensor_scale=1.0):
        if R.dtype != torch.float32 or R.dim() != 2 or R.stride(1) != 1:
            raise ValueError("expected a row-major 2-D fp32 CUDA tensor")
        q = QuantParams(rounding, seed, operand_id, step, tensor_scale)
        self._call(_quant_f32, _ptr(R), R.shape[0], R.shape[1], R.stride(0), ctypes.byref(q),
                   None if rowwise is None else ctypes.byref(rowwise.struct),
                   None if colwise is None else ctypes.byref(colwise.struct))

    def dequantize_nvfp4(self, t, out=None):
        """Decode an Nvfp4 tensor to fp32 (outer x inner) on the device."""
        if out is None:
            out = torch.empty(t.outer, t.inner, dtype=torch.float32, device=self.device)
        if out.dtype != torch.float32 or out.dim() != 2 or out.stride(1) != 1:
            raise ValueError("expected a row-major 2-D fp32 CUDA tensor")
        self._call(_dequant, ctypes.byref(t.struct), _ptr(out), out.stride(0))
        return out

    def gemm_nvfp4(self, A, B, n_cols, C, Fa=None, Fb=None, col_scale=None):
        fold_k = 0 if Fa is None else Fa.shape[1]
        dtype = OUT_F32 if C.dtype == torch.float32 else OUT_BF16
        self._call(_gemm, ctypes.byref(A.struct), ctypes.byref(B.struct), n_cols, _ptr(Fa), _ptr(Fb), fold_k,
                   _ptr(col_scale), _ptr(C), C.stride(0), dtype)

    def selftest_wait_timeout(self, limit_cycles=1_000_000):
        """Launch the bounded-wait self-test (a wait that must time out); the caller then
        reads METIS_DEV_TIMEOUT from poll_device_status()."""
        self._call(_wait_selftest, limit_cycles)

    def selftest_numeric(self):
        """Launch the numeric-latch self-test (an eigensolve allowed no sweep); the caller
        then reads METIS_DEV_NUMERIC from poll_device_status()."""
        self._call(_numeric_selftest)

    def nvfp4_mma_peak(self, iters=4096, reps=5):
        """Achievable NVFP4 MMA rate (TFLOP/s): the median of `reps` timed launches of the
        no-memory-traffic microbenchmark (after one untimed launch)."""
        fl = ctypes.c_double()
        self._call(_mma_peak, iters, ctypes.byref(fl))
        stream = torch.cuda.current_stream(self.device)
        times = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            self._call(_mma_peak, iters, ctypes.byref(fl))
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        times.sort()
        return fl.value / (times[len(times) // 2] * 1e-3) / 1e12

    def profile_enable(self, on=True):
        self._call(_prof_enable, int(bool(on)))

    def profile_read(self, kind=PROF_GEMM):
        """(milliseconds, launches, work) of the instrumented launches of one kind since the
        last read: flops for the main GeMM, algorithmic bytes for the residual quantizer
        and the projection."""
        ms, n, w = ctypes.c_double(), c_i64(), ctypes.c_double()
        self._call(_prof_read_kind, int(kind), ctypes.byref(ms), ctypes.byref(n), ctypes.byref(w))
        return ms.value, n.value, w.value

    @staticmethod
    def operand(rowwise=None, colwise=None, factors=None):
        return OperandStruct(None if rowwise is None else ctypes.pointer(rowwise.struct),
                             None if colwise is None else ctypes.pointer(colwise.struct),
                             None if factors is None else ctypes.pointer(factors.struct))

    def linear_fwd(self, X, W, Y):
        dtype = OUT_F32 if Y.dtype == torch.float32 else OUT_BF16
        self._call(_fwd, ctypes.byref(X), ctypes.byref(W), _ptr(Y), Y.stride(0), dtype)

    # -- LoRA-SVD linear projection (W = W_res + beta L2 L1) --------------------
    @staticmethod
    def _f32(t, name):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous fp32 CUDA tensor")
        return _ptr(t)

    def lora_linear(self, which, A, B, M, L2, L1, beta, C, T=None):
        """which 0: C = Q(X) Q(W_res) + beta (X L2) L1 (A = Q(X) row-wise, B = Q(W_res) column-wise,
        M = X); which 1: C = Q(D) Q(W_res)^T + beta (D L1^T) L2^T (A = Q(D) row-wise, B = Q(W_res)
        row-wise, M = D).  T (rows x k fp32, optional) receives X L2 or D L1^T."""
        dtype = OUT_F32 if C.dtype == torch.float32 else OUT_BF16
        self._call(_lora_linear, int(which), ctypes.byref(A.struct), ctypes.byref(B.struct),
                   ctypes.byref(_matrix(M)), self._f32(L2, "L2"), self._f32(L1, "L1"), L2.shape[1], float(beta),
                   None if T is None else self._f32(T, "T"), _ptr(C), C.stride(0), dtype)

    def lora_branch_grad(self, M, T, beta, G, transpose_out=False):
        """G = beta M^T T (cols x k), or its transpose (k x cols) with transpose_out."""
        self._call(_lora_grad, ctypes.byref(_matrix(M)), self._f32(T, "T"), T.shape[1], float(beta),
                   int(bool(transpose_out)), self._f32(G, "G"))

    def lora_constrain(self, L2, L1):
        """Cholesky-QR constraint in place: L2 = Q R -> L2 = Q, L1 = R L1."""
        self._call(_lora_constrain, self._f32(L2, "L2"), L2.shape[0], self._f32(L1, "L1"), L1.shape[1],
                   L2.shape[1])

    def lora_realign(self, W_res, L2, L1, beta, factors, W_bf16, s, l_k, seed, operand_id, step, rounding=0):
        """Randomized-SVD realignment in place (factors: m x n rank-k buffers; W_bf16: m x n scratch)."""
        k = L2.shape[1]
        p = DecompParams(k, s, l_k, seed, operand_id, rounding)
        if W_bf16.dtype != torch.bfloat16 or not W_bf16.is_contiguous():
            raise ValueError("W_bf16: expected a contiguous bf16 CUDA tensor")
        self._call(_lora_realign, self._f32(W_res, "W_res"), W_res.shape[0], W_res.shape[1], W_res.stride(0),
                   self._f32(L2, "L2"), self._f32(L1, "L1"), k, float(beta), ctypes.byref(p), int(step),
                   ctypes.byref(factors.struct), _ptr(W_bf16))

    def linear_bwd(self, X, W, D, dX, dW):
        dtype = OUT_F32 if dX.dtype == torch.float32 else OUT_BF16
        self._call(_bwd, ctypes.byref(X), ctypes.byref(W), ctypes.byref(D), _ptr(dX), dX.stride(0), dtype,
                   _ptr(dW), dW.stride(0))
