// The C ABI of libmetis: context management, host-side validation and dispatch.
#include <nvtx3/nvToolsExt.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <new>
#include <string>

#include "internal.h"

namespace metis {

// NVTX range over one C-ABI call (visible in profilers that record NVTX; near free otherwise).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

metis_status fail(metis_ctx* ctx, metis_status s, const std::string& msg) {
  if (ctx) ctx->last_error = msg;
  return s;
}

metis_status check_cuda(metis_ctx* ctx, cudaError_t e, const char* what) {
  if (e == cudaSuccess) return METIS_OK;
  return fail(ctx, METIS_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

metis_status ensure_workspace(metis_ctx* ctx, size_t bytes) {
  if (bytes <= ctx->ws_bytes) return METIS_OK;
  if (ctx->ws) {
    cudaStreamSynchronize(ctx->stream);
    cudaFree(ctx->ws);
    ctx->ws = nullptr;
    ctx->ws_bytes = 0;
  }
  const size_t want = (bytes + (size_t(1) << 20) - 1) & ~((size_t(1) << 20) - 1);
  if (cudaMalloc(&ctx->ws, want) != cudaSuccess) {
    cudaGetLastError();
    return fail(ctx, METIS_ERR_WORKSPACE, "could not allocate " + std::to_string(want) + " bytes of workspace");
  }
  ctx->ws_bytes = want;
  return METIS_OK;
}

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_positive(float g) {
  if (!(g > 0.0f) || !std::isfinite(g)) return false;
  int e;
  return std::frexp(g, &e) == 0.5f;
}

metis_status enter(metis_ctx* ctx) {
  if (!ctx) return METIS_ERR_ARG;
  ctx->last_error.clear();
  return check_cuda(ctx, cudaSetDevice(ctx->device), "cudaSetDevice");
}

metis_status check_nvfp4(metis_ctx* ctx, const metis_nvfp4* t, int64_t outer, int64_t inner, const char* name) {
  if (!t) return METIS_OK;
  if (!t->codes || !t->scales || !t->tensor_scale)
    return fail(ctx, METIS_ERR_ARG, std::string(name) + ": null codes, scales or tensor_scale");
  if (t->outer != outer || t->inner != inner)
    return fail(ctx, METIS_ERR_SHAPE, std::string(name) + ": expected outer x inner = " + std::to_string(outer) +
                                          " x " + std::to_string(inner));
  if (!aligned16(t->codes) || !aligned16(t->scales))
    return fail(ctx, METIS_ERR_ALIGN, std::string(name) + ": codes and scales must be 16-byte aligned");
  return METIS_OK;
}

metis_status check_dims(metis_ctx* ctx, int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0 || rows % 128 || cols % 128)
    return fail(ctx, METIS_ERR_SHAPE, "matrix dimensions must be positive multiples of 128");
  if (rows > (int64_t(1) << 31) || cols > (int64_t(1) << 31))
    return fail(ctx, METIS_ERR_SHAPE, "matrix dimension too large");
  return METIS_OK;
}

// The fused residual pass numbers its stochastic-rounding counters (element index / 16) in
// 32 bits: rows * cols <= 2^36 (a 128 GiB bf16 matrix).
metis_status check_fused_size(metis_ctx* ctx, int64_t rows, int64_t cols) {
  if ((double)rows * (double)cols > 68719476736.0)
    return fail(ctx, METIS_ERR_SHAPE, "rows * cols must not exceed 2^36 for the fused residual pass");
  return METIS_OK;
}

metis_status check_quant(metis_ctx* ctx, const metis_quant_params* q) {
  if (!q) return fail(ctx, METIS_ERR_ARG, "null quant params");
  if (q->rounding != 0 && q->rounding != 1) return fail(ctx, METIS_ERR_ARG, "rounding must be 0 (RN) or 1 (SR)");
  if (q->tensor_scale != 0.0f && !pow2_positive(q->tensor_scale))
    return fail(ctx, METIS_ERR_ARG, "tensor_scale must be a positive power of two, or 0 to choose it from the data");
  return METIS_OK;
}

}  // namespace

metis_status check_factors(metis_ctx* ctx, const metis_factors* f, int64_t rows, int64_t cols) {
  if (!f || f->k == 0) return METIS_OK;
  if (f->k < 0 || f->k > 64) return fail(ctx, METIS_ERR_SHAPE, "factor rank must be in [1, 64]");
  if (f->rows != rows || f->cols != cols) return fail(ctx, METIS_ERR_SHAPE, "factor shape does not match matrix");
  if (!f->U || !f->S || !f->V) return fail(ctx, METIS_ERR_ARG, "null factor buffer");
  if (!aligned16(f->U) || !aligned16(f->V)) return fail(ctx, METIS_ERR_ALIGN, "factor buffers must be 16-byte aligned");
  metis_status s = check_nvfp4(ctx, &f->Uq, 128, rows, "Uq");
  if (s != METIS_OK) return s;
  return check_nvfp4(ctx, &f->Vq, 128, cols, "Vq");
}

}  // namespace metis

using namespace metis;

extern "C" {

metis_status metis_create(int device, void* stream, metis_ctx** out) {
  if (!out) return METIS_ERR_ARG;
  *out = nullptr;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) {
    cudaGetLastError();
    return METIS_ERR_CUDA;
  }
  if (prop.major != 10 || prop.minor != 0) return METIS_ERR_ARCH;
  if (cudaSetDevice(device) != cudaSuccess) return METIS_ERR_CUDA;
  metis_ctx* ctx = new (std::nothrow) metis_ctx();
  if (!ctx) return METIS_ERR_WORKSPACE;
  ctx->device = device;
  ctx->stream = static_cast<cudaStream_t>(stream);
  ctx->sm_count = prop.multiProcessorCount;
  ctx->sm_count_device = prop.multiProcessorCount;
  if (cudaMalloc(&ctx->status, sizeof(uint32_t)) != cudaSuccess || cudaMemset(ctx->status, 0, sizeof(uint32_t)) != cudaSuccess) {
    delete ctx;
    return METIS_ERR_CUDA;
  }
  if (!encode_tiled()) {
    cudaFree(ctx->status);
    delete ctx;
    return METIS_ERR_CUDA;
  }
  *out = ctx;
  return METIS_OK;
}

void metis_destroy(metis_ctx* ctx) {
  if (!ctx) return;
  cudaSetDevice(ctx->device);
  cudaStreamSynchronize(ctx->stream);
  if (ctx->ws) cudaFree(ctx->ws);
  if (ctx->status) cudaFree(ctx->status);
  for (auto& evs : ctx->prof_events)
    for (auto& ev : evs) {
      cudaEventDestroy(ev.first);
      cudaEventDestroy(ev.second);
    }
  delete ctx;
}

metis_status metis_set_stream(metis_ctx* ctx, void* stream) {
  if (!ctx) return METIS_ERR_ARG;
  ctx->stream = static_cast<cudaStream_t>(stream);
  return METIS_OK;
}

metis_status metis_set_sm_count_target(metis_ctx* ctx, int n) {
  if (!ctx) return METIS_ERR_ARG;
  if (n < 0 || n > ctx->sm_count_device || (n > 0 && n < 2))
    return fail(ctx, METIS_ERR_ARG, "SM count target must be 0 or between 2 and the device's SM count");
  ctx->sm_count = n == 0 ? ctx->sm_count_device : n;
  return METIS_OK;
}

const char* metis_status_str(metis_status s) {
  switch (s) {
    case METIS_OK: return "ok";
    case METIS_ERR_ARG: return "invalid argument";
    case METIS_ERR_SHAPE: return "unsupported shape";
    case METIS_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case METIS_ERR_ARCH: return "device is not sm_100 (B200)";
    case METIS_ERR_CUDA: return "CUDA error";
    case METIS_ERR_WORKSPACE: return "workspace allocation failed";
  }
  return "unknown status";
}

const char* metis_last_error(const metis_ctx* ctx) { return ctx ? ctx->last_error.c_str() : "null context"; }

metis_status metis_poll_device_status(metis_ctx* ctx, uint32_t* bits, int clear) {
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!bits) return fail(ctx, METIS_ERR_ARG, "null bits");
  s = check_cuda(ctx, cudaStreamSynchronize(ctx->stream), "cudaStreamSynchronize");
  if (s != METIS_OK) return s;
  s = check_cuda(ctx, cudaMemcpy(bits, ctx->status, sizeof(uint32_t), cudaMemcpyDeviceToHost), "status read");
  if (s != METIS_OK) return s;
  if (clear) s = check_cuda(ctx, cudaMemset(ctx->status, 0, sizeof(uint32_t)), "status clear");
  return s;
}

int64_t metis_nvfp4_codes_bytes(int64_t outer, int64_t inner) { return outer * inner / 2; }

int64_t metis_nvfp4_scales_bytes(int64_t outer, int64_t inner) {
  return ((outer + 127) / 128) * ((inner + 63) / 64) * 512;
}

metis_status metis_quantize_nvfp4_f32(metis_ctx* ctx, const float* R, int64_t rows, int64_t cols, int64_t ld,
                                      const metis_quant_params* q, metis_nvfp4* rowwise, metis_nvfp4* colwise) {
  const metis::NvtxRange nvtx_range("metis_quantize_nvfp4_f32");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!R) return fail(ctx, METIS_ERR_ARG, "null input");
  if ((s = check_dims(ctx, rows, cols)) != METIS_OK) return s;
  if (ld < cols || ld % 4 || !aligned16(R)) return fail(ctx, METIS_ERR_ALIGN, "fp32 input needs 16-byte alignment and ld % 4 == 0");
  if ((s = check_quant(ctx, q)) != METIS_OK) return s;
  if (!rowwise && !colwise) return fail(ctx, METIS_ERR_ARG, "no output orientation requested");
  if ((s = check_nvfp4(ctx, rowwise, rows, cols, "rowwise")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, colwise, cols, rows, "colwise")) != METIS_OK) return s;
  uint32_t* amax = nullptr;
  if (q->tensor_scale == 0.0f) {
    if ((s = ensure_workspace(ctx, 256)) != METIS_OK) return s;
    amax = reinterpret_cast<uint32_t*>(ctx->ws);
    if ((s = check_cuda(ctx, launch_amax(R, false, rows, cols, ld, amax, ctx->sm_count, ctx->stream),
                        "amax launch")) != METIS_OK)
      return s;
  }
  return check_cuda(ctx,
                    launch_quantize_f32(R, rows, cols, ld, *q, amax, rowwise, colwise, ctx->status, ctx->stream),
                    "quantize launch");
}

metis_status metis_dequantize_nvfp4(metis_ctx* ctx, const metis_nvfp4* t, float* out, int64_t ld) {
  const metis::NvtxRange nvtx_range("metis_dequantize_nvfp4");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!t || !out) return fail(ctx, METIS_ERR_ARG, "null tensor or output");
  if ((s = check_nvfp4(ctx, t, t->outer, t->inner, "tensor")) != METIS_OK) return s;
  if (t->outer <= 0 || t->inner <= 0 || t->inner % 64) return fail(ctx, METIS_ERR_SHAPE, "inner must be a multiple of 64");
  if (ld < t->inner || ld % 4 || !aligned16(out))
    return fail(ctx, METIS_ERR_ALIGN, "fp32 output needs 16-byte alignment and ld % 4 == 0");
  return check_cuda(ctx, launch_dequantize(t, out, ld, ctx->stream), "dequantize launch");
}

metis_status metis_residual_quantize_nvfp4(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                           const metis_quant_params* q, metis_nvfp4* rowwise,
                                           metis_nvfp4* colwise) {
  const metis::NvtxRange nvtx_range("metis_residual_quantize_nvfp4");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!M || !M->data) return fail(ctx, METIS_ERR_ARG, "null matrix");
  if ((s = check_dims(ctx, M->rows, M->cols)) != METIS_OK) return s;
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if ((s = check_quant(ctx, q)) != METIS_OK) return s;
  if ((s = check_factors(ctx, f, M->rows, M->cols)) != METIS_OK) return s;
  if (!rowwise && !colwise) return fail(ctx, METIS_ERR_ARG, "no output orientation requested");
  if ((s = check_nvfp4(ctx, rowwise, M->rows, M->cols, "rowwise")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, colwise, M->cols, M->rows, "colwise")) != METIS_OK) return s;
  if (rowwise && colwise) {
    if ((s = check_fused_size(ctx, M->rows, M->cols)) != METIS_OK) return s;
    return run_residual_quantize(ctx, M, f, q, rowwise, colwise);
  }
  // one orientation only: fp32 residual in the workspace, then the quantizer
  const size_t bytes = (size_t)M->rows * M->cols * sizeof(float);
  if ((s = ensure_workspace(ctx, bytes + 512)) != METIS_OK) return s;
  float* R = reinterpret_cast<float*>(ctx->ws);
  uint32_t* amax = nullptr;
  if (q->tensor_scale == 0.0f) {   // g from the amax of M, as in the two-orientation path
    amax = reinterpret_cast<uint32_t*>(ctx->ws + ((bytes + 255) & ~size_t(255)));
    if ((s = check_cuda(ctx, launch_amax(M->data, true, M->rows, M->cols, M->ld, amax, ctx->sm_count, ctx->stream),
                        "amax launch")) != METIS_OK)
      return s;
  }
  const bool lowrank = f && f->k > 0;
  s = check_cuda(ctx,
                 launch_residual_f32(M->data, M->rows, M->cols, M->ld, lowrank ? f->U : nullptr,
                                     lowrank ? f->S : nullptr, lowrank ? f->V : nullptr, lowrank ? f->k : 0, R,
                                     ctx->status, ctx->stream),
                 "residual launch");
  if (s != METIS_OK) return s;
  return check_cuda(ctx,
                    launch_quantize_f32(R, M->rows, M->cols, M->cols, *q, amax, rowwise, colwise, ctx->status,
                                        ctx->stream),
                    "quantize launch");
}

metis_status metis_residual_quantize_nvfp4_dump(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                                const metis_quant_params* q, metis_nvfp4* rowwise,
                                                metis_nvfp4* colwise, float* residual, int64_t ldr) {
  const metis::NvtxRange nvtx_range("metis_residual_quantize_nvfp4_dump");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!M || !M->data) return fail(ctx, METIS_ERR_ARG, "null matrix");
  if ((s = check_dims(ctx, M->rows, M->cols)) != METIS_OK) return s;
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if ((s = check_quant(ctx, q)) != METIS_OK) return s;
  if ((s = check_factors(ctx, f, M->rows, M->cols)) != METIS_OK) return s;
  if (!rowwise || !colwise || !residual) return fail(ctx, METIS_ERR_ARG, "both orientations and the residual are required");
  if ((s = check_nvfp4(ctx, rowwise, M->rows, M->cols, "rowwise")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, colwise, M->cols, M->rows, "colwise")) != METIS_OK) return s;
  if (ldr < M->cols || ldr % 4 || !aligned16(residual))
    return fail(ctx, METIS_ERR_ALIGN, "fp32 residual needs 16-byte alignment and ld % 4 == 0");
  if ((s = check_fused_size(ctx, M->rows, M->cols)) != METIS_OK) return s;
  return run_residual_quantize(ctx, M, f, q, rowwise, colwise, residual, ldr);
}

metis_status metis_gemm_nvfp4(metis_ctx* ctx, const metis_nvfp4* A, const metis_nvfp4* B, int64_t n_cols,
                              const void* Fa, const void* Fb, int32_t fold_k, const float* col_scale, void* C,
                              int64_t ldc, int32_t c_dtype) {
  const metis::NvtxRange nvtx_range("metis_gemm_nvfp4");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!A || !B || !C) return fail(ctx, METIS_ERR_ARG, "null operand");
  if (A->inner != B->inner || A->inner <= 0 || A->inner % 256)
    return fail(ctx, METIS_ERR_SHAPE, "A.inner must equal B.inner and be a multiple of 256");
  if (A->outer <= 0 || A->outer % 128) return fail(ctx, METIS_ERR_SHAPE, "A.outer must be a multiple of 128");
  const bool thin = n_cols == 16 || n_cols == 32 || n_cols == 64;
  if (!thin && (n_cols <= 0 || n_cols % 256 || B->outer != n_cols))
    return fail(ctx, METIS_ERR_SHAPE, "n_cols must be a multiple of 256 equal to B.outer, or 16/32/64");
  if (thin && B->outer != 128) return fail(ctx, METIS_ERR_SHAPE, "a thin GeMM needs B.outer == 128 (zero-padded)");
  if ((s = check_nvfp4(ctx, A, A->outer, A->inner, "A")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, B, B->outer, B->inner, "B")) != METIS_OK) return s;
  if (fold_k < 0 || fold_k % 64) return fail(ctx, METIS_ERR_SHAPE, "fold_k must be a non-negative multiple of 64");
  if (fold_k > 0 && (!Fa || !Fb)) return fail(ctx, METIS_ERR_ARG, "fold operands missing");
  if (fold_k > 0 && (!aligned16(Fa) || !aligned16(Fb))) return fail(ctx, METIS_ERR_ALIGN, "fold operands must be 16-byte aligned");
  if (c_dtype != METIS_OUT_F32 && c_dtype != METIS_OUT_BF16) return fail(ctx, METIS_ERR_ARG, "bad output dtype");
  if (ldc < n_cols || ldc % (c_dtype == METIS_OUT_F32 ? 4 : 8) || !aligned16(C))
    return fail(ctx, METIS_ERR_ALIGN, "output needs 16-byte alignment and a 16-byte multiple leading dimension");
  GemmArgs a{A, B, fold_k ? Fa : nullptr, fold_k ? Fb : nullptr, fold_k, col_scale, C, ldc, c_dtype, 1.0f, n_cols, 1, 0};
  return launch_gemm_nvfp4(ctx, a);
}

metis_status metis_decompose(metis_ctx* ctx, const metis_matrix* M, const metis_decomp_params* p, int refresh,
                             uint32_t step, metis_factors* f) {
  const metis::NvtxRange nvtx_range("metis_decompose");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!M || !M->data || !p || !f) return fail(ctx, METIS_ERR_ARG, "null argument");
  if ((s = check_dims(ctx, M->rows, M->cols)) != METIS_OK) return s;
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if (p->k < 1 || p->k > 64 || p->s < 0 || p->k + p->s > 128 || p->l_k < p->k + p->s || p->l_k > M->rows ||
      p->k + p->s > M->cols)
    return fail(ctx, METIS_ERR_SHAPE, "need 1 <= k <= 64, k + s <= 128, k + s <= l_k <= rows, k + s <= cols");
  if (p->rounding != 0 && p->rounding != 1) return fail(ctx, METIS_ERR_ARG, "rounding must be 0 or 1");
  if (f->k != p->k) return fail(ctx, METIS_ERR_SHAPE, "factors.k != params.k");
  if ((s = check_factors(ctx, f, M->rows, M->cols)) != METIS_OK) return s;
  return run_decompose(ctx, M, p, refresh, step, f);
}

metis_status metis_linear_fwd(metis_ctx* ctx, const metis_operand* X, const metis_operand* W, void* Y, int64_t ldy,
                              int32_t y_dtype) {
  const metis::NvtxRange nvtx_range("metis_linear_fwd");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!X || !W || !Y || !X->rowwise || !W->colwise) return fail(ctx, METIS_ERR_ARG, "null operand");
  return run_linear(ctx, X, X->rowwise, W, W->colwise, false, false, Y, ldy, y_dtype);
}

metis_status metis_linear_bwd(metis_ctx* ctx, const metis_operand* X, const metis_operand* W, const metis_operand* D,
                              void* dX, int64_t lddx, int32_t dx_dtype, float* dW, int64_t lddw) {
  const metis::NvtxRange nvtx_range("metis_linear_bwd");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!X || !W || !D || !dX || !dW || !D->rowwise || !D->colwise || !W->rowwise || !X->colwise)
    return fail(ctx, METIS_ERR_ARG, "null operand");
  // dX = D_hat W_hat^T: the B operand is W^T, whose factors swap roles (V, S, U)
  s = run_linear(ctx, D, D->rowwise, W, W->rowwise, false, true, dX, lddx, dx_dtype);
  if (s != METIS_OK) return s;
  // dW = X_hat^T D_hat: the A operand is X^T (factors B, L, A)
  return run_linear(ctx, X, X->colwise, D, D->colwise, true, false, dW, lddw, METIS_OUT_F32);
}

metis_status metis_lora_linear(metis_ctx* ctx, int32_t which, const metis_nvfp4* A, const metis_nvfp4* B,
                               const metis_matrix* M, const float* L2, const float* L1, int32_t k, float beta,
                               float* T, void* C, int64_t ldc, int32_t c_dtype) {
  const metis::NvtxRange nvtx_range("metis_lora_linear");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (which != 0 && which != 1) return fail(ctx, METIS_ERR_ARG, "which must be 0 (forward) or 1 (input gradient)");
  if (!A || !B || !M || !M->data || !L2 || !L1 || !C) return fail(ctx, METIS_ERR_ARG, "null argument");
  if (k < 1 || k > 64) return fail(ctx, METIS_ERR_SHAPE, "LoRA rank must be in [1, 64]");
  if (!std::isfinite(beta)) return fail(ctx, METIS_ERR_ARG, "beta must be finite");
  const int64_t p = A->outer, K = A->inner, q = B->outer;
  if (B->inner != K || K <= 0 || K % 256) return fail(ctx, METIS_ERR_SHAPE, "A.inner must equal B.inner and be a multiple of 256");
  if ((s = check_dims(ctx, p, K)) != METIS_OK) return s;
  if (q <= 0 || q % 256) return fail(ctx, METIS_ERR_SHAPE, "B.outer (the output columns) must be a multiple of 256");
  if ((s = check_nvfp4(ctx, A, p, K, "A")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, B, q, K, "B")) != METIS_OK) return s;
  if (M->rows != p || M->cols != K) return fail(ctx, METIS_ERR_SHAPE, "M must be A.outer x A.inner");
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if (c_dtype != METIS_OUT_F32 && c_dtype != METIS_OUT_BF16) return fail(ctx, METIS_ERR_ARG, "bad output dtype");
  if (ldc < q || ldc % (c_dtype == METIS_OUT_F32 ? 4 : 8) || !aligned16(C))
    return fail(ctx, METIS_ERR_ALIGN, "output needs 16-byte alignment and a 16-byte multiple leading dimension");
  if (!aligned16(L2) || !aligned16(L1) || (T && !aligned16(T)))
    return fail(ctx, METIS_ERR_ALIGN, "L2, L1 and T must be 16-byte aligned");
  return run_lora_linear(ctx, which, A, B, M, L2, L1, k, beta, T, C, ldc, c_dtype);
}

metis_status metis_lora_branch_grad(metis_ctx* ctx, const metis_matrix* M, const float* T, int32_t k, float beta,
                                    int32_t transpose_out, float* G) {
  const metis::NvtxRange nvtx_range("metis_lora_branch_grad");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!M || !M->data || !T || !G) return fail(ctx, METIS_ERR_ARG, "null argument");
  if (k < 1 || k > 64) return fail(ctx, METIS_ERR_SHAPE, "LoRA rank must be in [1, 64]");
  if (!std::isfinite(beta)) return fail(ctx, METIS_ERR_ARG, "beta must be finite");
  if ((s = check_dims(ctx, M->rows, M->cols)) != METIS_OK) return s;
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if (!aligned16(T) || !aligned16(G)) return fail(ctx, METIS_ERR_ALIGN, "T and G must be 16-byte aligned");
  return run_lora_branch_grad(ctx, M, T, k, beta, transpose_out != 0, G);
}

metis_status metis_lora_constrain(metis_ctx* ctx, float* L2, int64_t m, float* L1, int64_t n, int32_t k) {
  const metis::NvtxRange nvtx_range("metis_lora_constrain");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!L2 || !L1) return fail(ctx, METIS_ERR_ARG, "null argument");
  if (k < 1 || k > 64) return fail(ctx, METIS_ERR_SHAPE, "LoRA rank must be in [1, 64]");
  if ((s = check_dims(ctx, m, n)) != METIS_OK) return s;
  if (!aligned16(L2) || !aligned16(L1)) return fail(ctx, METIS_ERR_ALIGN, "L2 and L1 must be 16-byte aligned");
  return run_lora_constrain(ctx, L2, m, L1, n, k);
}

metis_status metis_lora_realign(metis_ctx* ctx, float* W_res, int64_t m, int64_t n, int64_t ldw, float* L2,
                                float* L1, int32_t k, float beta, const metis_decomp_params* p, uint32_t step,
                                metis_factors* f, void* W_bf16) {
  const metis::NvtxRange nvtx_range("metis_lora_realign");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!W_res || !L2 || !L1 || !p || !f || !W_bf16) return fail(ctx, METIS_ERR_ARG, "null argument");
  if (!(std::isfinite(beta) && beta != 0.0f)) return fail(ctx, METIS_ERR_ARG, "beta must be finite and nonzero");
  if ((s = check_dims(ctx, m, n)) != METIS_OK) return s;
  if (ldw < n || ldw % 4 || !aligned16(W_res) || !aligned16(W_bf16) || !aligned16(L2) || !aligned16(L1))
    return fail(ctx, METIS_ERR_ALIGN, "W_res, W_bf16, L2, L1 need 16-byte alignment and ldw % 4 == 0");
  if (k < 1 || k > 64 || p->k != k || f->k != k)
    return fail(ctx, METIS_ERR_SHAPE, "LoRA rank must be in [1, 64] and equal params.k and factors.k");
  if (p->s < 0 || p->k + p->s > 128 || p->l_k < p->k + p->s || p->l_k > m || p->k + p->s > n)
    return fail(ctx, METIS_ERR_SHAPE, "need k + s <= 128, k + s <= l_k <= m, k + s <= n");
  if (p->rounding != 0 && p->rounding != 1) return fail(ctx, METIS_ERR_ARG, "rounding must be 0 or 1");
  if ((s = check_factors(ctx, f, m, n)) != METIS_OK) return s;
  return run_lora_realign(ctx, W_res, m, n, ldw, L2, L1, k, beta, p, step, f, W_bf16);
}

}  // extern "C"

namespace metis {
std::atomic<uint64_t> g_launches{0};

void profile_record(metis_ctx* ctx, int kind, cudaEvent_t ev0, cudaEvent_t ev1, double work) {
  ctx->prof_events[kind].emplace_back(ev0, ev1);
  ctx->prof_work[kind].push_back(work);
}
}  // namespace metis

extern "C" {

uint64_t metis_kernel_launches(void) { return metis::g_launches.load(); }

metis_status metis_profile_enable(metis_ctx* ctx, int on) {
  if (!ctx) return METIS_ERR_ARG;
  ctx->profiling = on != 0;
  return METIS_OK;
}

metis_status metis_selftest_wait_timeout(metis_ctx* ctx, int64_t limit_cycles) {
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (limit_cycles < 1 || limit_cycles > 200000000LL)
    return fail(ctx, METIS_ERR_ARG, "limit_cycles must be in [1, 2e8]");
  return launch_wait_timeout_selftest(ctx, limit_cycles);
}

metis_status metis_selftest_numeric(metis_ctx* ctx) {
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  return launch_numeric_selftest(ctx);
}

metis_status metis_nvfp4_mma_peak(metis_ctx* ctx, int64_t iters, double* flops) {
  const metis::NvtxRange nvtx_range("metis_nvfp4_mma_peak");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!flops || iters < 1 || iters > (int64_t(1) << 20))
    return fail(ctx, METIS_ERR_ARG, "iters must be in [1, 2^20] and flops non-null");
  return launch_mma_peak(ctx, iters, flops);
}

metis_status metis_profile_read_kind(metis_ctx* ctx, int32_t kind, double* ms, int64_t* launches, double* work) {
  if (!ctx || !ms || !launches || !work || kind < 0 || kind >= metis::kProfKinds) return METIS_ERR_ARG;
  cudaSetDevice(ctx->device);
  metis_status s = metis::check_cuda(ctx, cudaStreamSynchronize(ctx->stream), "cudaStreamSynchronize");
  if (s != METIS_OK) return s;
  auto& evs = ctx->prof_events[kind];
  auto& wk = ctx->prof_work[kind];
  double total = 0.0, w = 0.0;
  for (size_t i = 0; i < evs.size(); ++i) {
    float t = 0.0f;
    cudaEventElapsedTime(&t, evs[i].first, evs[i].second);
    total += t;
    w += wk[i];
    cudaEventDestroy(evs[i].first);
    cudaEventDestroy(evs[i].second);
  }
  *ms = total;
  *launches = (int64_t)evs.size();
  *work = w;
  evs.clear();
  wk.clear();
  return METIS_OK;
}

metis_status metis_profile_read(metis_ctx* ctx, double* ms, int64_t* launches, double* flops) {
  return metis_profile_read_kind(ctx, METIS_PROF_GEMM, ms, launches, flops);
}

}  // extern "C"

extern "C" metis_status metis_residual_quantize_nvfp4_noalloc(metis_ctx* ctx, const metis_matrix* M,
                                                               const metis_factors* f, const metis_quant_params* q,
                                                               metis_nvfp4* rowwise, metis_nvfp4* colwise) {
  const metis::NvtxRange nvtx_range("metis_residual_quantize_nvfp4_noalloc");
  metis_status s = enter(ctx);
  if (s != METIS_OK) return s;
  if (!M || !M->data) return fail(ctx, METIS_ERR_ARG, "null matrix");
  if ((s = check_dims(ctx, M->rows, M->cols)) != METIS_OK) return s;
  if (M->rows + M->cols > kNoAllocMaxRowsPlusCols)
    return fail(ctx, METIS_ERR_SHAPE, "rows + cols = " + std::to_string(M->rows + M->cols) +
                                          " exceeds the allocation-free limit of " +
                                          std::to_string(kNoAllocMaxRowsPlusCols));
  if (M->ld < M->cols || M->ld % 8 || !aligned16(M->data))
    return fail(ctx, METIS_ERR_ALIGN, "bf16 matrix needs 16-byte alignment and ld % 8 == 0");
  if ((s = check_quant(ctx, q)) != METIS_OK) return s;
  if ((s = check_factors(ctx, f, M->rows, M->cols)) != METIS_OK) return s;
  if (!rowwise || !colwise) return fail(ctx, METIS_ERR_ARG, "the allocation-free path writes both orientations");
  if ((s = check_nvfp4(ctx, rowwise, M->rows, M->cols, "rowwise")) != METIS_OK) return s;
  if ((s = check_nvfp4(ctx, colwise, M->cols, M->rows, "colwise")) != METIS_OK) return s;
  char* scratch = noalloc_scratch(ctx, &s);
  if (!scratch) return s;
  if (residual_quantize_scratch_bytes(M->rows, M->cols) > kNoAllocAmaxOffset)
    return fail(ctx, METIS_ERR_SHAPE, "shape needs more than the allocation-free scratch");
  return run_residual_quantize_into(ctx, M, f, q, rowwise, colwise, scratch,
                                    reinterpret_cast<uint32_t*>(scratch + kNoAllocAmaxOffset), nullptr, 0);
}
