// Host-side internals of libmetis: the context, workspace and kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <string>
#include <vector>

#include "../../include/metis.h"

struct metis_ctx {
  int device = 0;
  cudaStream_t stream = nullptr;
  int sm_count = 0;            // SMs the persistent grids and split counts are sized for
  int sm_count_device = 0;     // the device's SM count
  uint32_t* status = nullptr;  // device status word (METIS_DEV_* bits)
  char* ws = nullptr;          // device workspace, grown on demand
  size_t ws_bytes = 0;
  std::string last_error;
  bool profiling = false;
  // per instrumented kernel kind (metis::kProf*): event pairs around each launch and the
  // launch's algorithmic work (flops or bytes)
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof_events[3];
  std::vector<double> prof_work[3];
};

namespace metis {

// Process-wide count of kernels launched by libmetis.
extern std::atomic<uint64_t> g_launches;
inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Kernels bracketed by CUDA events while profiling is on (metis_profile_read_kind).
enum : int { kProfGemm = 0, kProfResquant = 1, kProfProjection = 2, kProfKinds = 3 };
// Records one launch of `kind` between events ev0 and ev1 (already recorded on ctx->stream).
void profile_record(metis_ctx* ctx, int kind, cudaEvent_t ev0, cudaEvent_t ev1, double work);

// Sub-allocator over the context workspace: hands out 256-byte aligned slices.
struct Workspace {
  char* base;
  size_t cap;
  size_t used = 0;
  void* take(size_t bytes) {
    size_t off = (used + 255) & ~size_t(255);
    if (off + bytes > cap) return nullptr;
    used = off + bytes;
    return base + off;
  }
};

metis_status ensure_workspace(metis_ctx* ctx, size_t bytes);
metis_status fail(metis_ctx* ctx, metis_status s, const std::string& msg);
metis_status check_cuda(metis_ctx* ctx, cudaError_t e, const char* what);

// cuTensorMapEncodeTiled, fetched from the driver through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// ---- quantize.cu ----
// Decode tensor scale chosen from the data (metis_quant_params.tensor_scale == 0):
// launch_amax writes max |x| over the finite entries of M (bf16 or fp32, row-major) as
// fp32 bits to *amax_bits; the quantizers then take g = auto_tensor_scale(*amax_bits).
cudaError_t launch_amax(const void* M, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax_bits,
                        int sm_count, cudaStream_t st);
// Decode of one NVFP4 tensor into fp32 (outer x inner, leading dimension ld).
cudaError_t launch_dequantize(const metis_nvfp4* t, float* out, int64_t ld, cudaStream_t st);
// amax_bits: nullptr to use q.tensor_scale, else the word launch_amax wrote.
cudaError_t launch_quantize_f32(const float* R, int64_t rows, int64_t cols, int64_t ld,
                                const metis_quant_params& q, const uint32_t* amax_bits, const metis_nvfp4* rowwise,
                                const metis_nvfp4* colwise, uint32_t* status, cudaStream_t st);
cudaError_t launch_residual_f32(const void* M_bf16, int64_t rows, int64_t cols, int64_t ld, const float* U,
                                const float* S, const float* V, int32_t k, float* out, uint32_t* status,
                                cudaStream_t st);

// ---- resquant.cu ----
// Both orientations in one pass over M; `residual` (nullable, fp32, leading dimension ld_res)
// receives the residual the quantizer rounded.  Scratch in the context workspace.
metis_status run_residual_quantize(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                   const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col,
                                   float* residual = nullptr, int64_t ld_res = 0);
// Device scratch the pass needs besides the amax word: the fp16 hi/lo factor tiles and
// their per-block power-of-two factors.
size_t residual_quantize_scratch_bytes(int64_t rows, int64_t cols);
// The same pass with caller-provided scratch (residual_quantize_scratch_bytes(rows, cols)
// bytes, 256-byte aligned) and amax word (used when q->tensor_scale == 0).
metis_status run_residual_quantize_into(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                        const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col,
                                        void* scratch, uint32_t* amax_word, float* residual, int64_t ld_res);

// ---- noalloc.cu ----
// Limits of the allocation-free residual quantizer's fixed scratch: the factor tiles and
// block factors of residual_quantize_scratch_bytes for rows + cols <= 24576 (256 bytes
// per row or column, at most 1 KiB of block factors), then 256 bytes whose first word
// holds the amax of a call that asks for a tensor scale chosen from the data.
constexpr int64_t kNoAllocMaxRowsPlusCols = 24576;
constexpr size_t kNoAllocAmaxOffset = (size_t)kNoAllocMaxRowsPlusCols * 256 + 1024;   // bytes
constexpr size_t kNoAllocBytes = kNoAllocAmaxOffset + 256;
char* noalloc_scratch(metis_ctx* ctx, metis_status* st);

// ---- gemm_fp4.cu ----
struct GemmArgs {
  const metis_nvfp4* A;
  const metis_nvfp4* B;
  const void* Fa;
  const void* Fb;
  int32_t fold_k;
  const float* col_scale;
  void* C;
  int64_t ldc;
  int32_t c_dtype;
  float alpha_extra;  // multiplies alpha = gA * gB (1.0 normally)
  int64_t q_cols;     // output columns: a multiple of 256, or 16 / 32 / 64 (thin)
  int32_t k_splits;       // > 1: split-K over the FP4 + fold stages, partial s at C + s * split_stride (fp32)
  int64_t split_stride;   // elements between consecutive partial outputs
};
// Split count for an FP4 GeMM of `tiles` output tiles and `stages` K stages (no empty
// share): the one whose units fill the persistent grid's rounds best.
int fp4_splits(metis_ctx* ctx, int64_t tiles, int stages);
metis_status launch_gemm_nvfp4(metis_ctx* ctx, const GemmArgs& a);
// Up to three thin GeMMs (the same width 16/32/64 and K, fp32 outputs, no fold) in one launch.
metis_status launch_gemm_nvfp4_group(metis_ctx* ctx, const GemmArgs* g, int n);
// ---- selftest.cu ----
metis_status launch_wait_timeout_selftest(metis_ctx* ctx, int64_t limit_cycles);
// (decompose.cu) the eigensolver on a fixed 8 x 8 matrix with a sweep limit of zero
metis_status launch_numeric_selftest(metis_ctx* ctx);
// ---- mma_peak.cu ----
metis_status launch_mma_peak(metis_ctx* ctx, int64_t iters, double* flops);
// Split count for a bf16 GeMM of rows / 128 tiles, K / 64 stages and output width n,
// chosen the same way, with the cost of each split's partials counted.
int bf16_splits(metis_ctx* ctx, int64_t rows, int64_t K, int n);
// Split count with no empty share of the K / 64 stages (what the launch uses).
inline int normalize_splits(int64_t K, int splits) {
  const int stages = (int)(K / 64);
  const int per = (stages + splits - 1) / splits;
  return (stages + per - 1) / per;
}
// C[s] (rows x n, fp32, split s at C + s * rows * ldc) = A (rows x K bf16, lda) * B^T
// (B: n x K bf16, ldb) over the s-th share of K.  splits < 1 picks a split count.
metis_status launch_gemm_bf16(metis_ctx* ctx, const void* A, int64_t lda, int64_t rows, const void* B, int64_t ldb,
                              int n, int64_t K, float* C, int64_t ldc, int splits);

// ---- decompose.cu ----
metis_status run_decompose(metis_ctx* ctx, const metis_matrix* M, const metis_decomp_params* p, int refresh,
                           uint32_t step, metis_factors* f);

// Shared with lora.cu.  Mt (c x r bf16) = M^T for M (r x c bf16, leading dimension ld),
// r and c multiples of 64.
cudaError_t launch_transpose_bf16(const void* M, int64_t ld, int64_t r, int64_t c, void* Mt, cudaStream_t st);
// out (2 kp x n bf16) = [F^T hi ; F^T lo] for F (n x k fp32), rows k .. kp - 1 of each half zero.
cudaError_t launch_split_hi_lo_t(const float* F, int64_t n, int k, int kp, void* out, cudaStream_t st);
// G = A^T A (fp64, w x w, full) of a tall fp32 matrix A (n x w, row-major, w <= 64),
// deterministic; G lives in `scratch` (gram_scratch_doubles(ctx, w) doubles).
size_t gram_scratch_doubles(metis_ctx* ctx, int w);
metis_status launch_gram(metis_ctx* ctx, const float* A, int64_t n, int w, double* scratch, double** G_out);

// ---- lora.cu ----
metis_status run_lora_linear(metis_ctx* ctx, int which, const metis_nvfp4* A, const metis_nvfp4* B,
                             const metis_matrix* M, const float* L2, const float* L1, int k, float beta, float* T,
                             void* C, int64_t ldc, int32_t c_dtype);
metis_status run_lora_branch_grad(metis_ctx* ctx, const metis_matrix* M, const float* T, int k, float beta,
                                  bool transpose_out, float* G);
metis_status run_lora_constrain(metis_ctx* ctx, float* L2, int64_t m, float* L1, int64_t n, int k);
metis_status run_lora_realign(metis_ctx* ctx, float* W, int64_t m, int64_t n, int64_t ldw, float* L2, float* L1,
                              int k, float beta, const metis_decomp_params* p, uint32_t step, metis_factors* f,
                              void* W_bf16);

// ---- layer.cu ----
metis_status run_linear(metis_ctx* ctx, const metis_operand* A, const metis_nvfp4* A_res, const metis_operand* B,
                        const metis_nvfp4* B_res, bool a_transposed_factors, bool b_transposed_factors, void* C,
                        int64_t ldc, int32_t c_dtype);

}  // namespace metis
