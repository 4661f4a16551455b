// The Metis linear layer: fold preparation and the fused GeMM.
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
// key design 1 (forward equation) and framework section (the split is used in
// every forward and backward GeMM).  For C = A_hat B_hat with
//   A_hat = Q(L_A) S_A Q(R_A)^T + Q(A_R),   B_hat = Q(L_B) S_B Q(R_B)^T + Q(B_R)
// the product is evaluated as
//   C = Q(A_R) Q(B_R) + Q(L_A) T_A + T_B Q(R_B)^T
//   T_A = S_A Q(R_A)^T (Q(B_R) + Q(L_B) S_B Q(R_B)^T)      (k_A x q)
//   T_B = Q(A_R) Q(L_B) S_B                                (p x k_B)
// T_A and T_B are kept at ~16-bit precision as bf16 hi + lo pairs, so the fold
// operands are
//   Fa = [Q(L_A) | Q(L_A) | T_B hi | T_B lo] / alpha,   Fb = [T_A^T hi | T_A^T lo | Q(R_B) | Q(R_B)]
// with alpha = gA * gB the tensor-scale product of the main FP4 GeMM, and one
// fused kernel computes C = alpha * (Q(A_R) Q(B_R) + Fa Fb^T).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"

namespace metis {
namespace {

// Decoded value of element (row t, column i) of a k x len factor NVFP4 tensor
// (the transposed storage of a len x k factor).
__device__ __forceinline__ float factor_value(const uint8_t* codes, const uint8_t* scales, float g, int64_t len,
                                              int t, int64_t i) {
  const uint8_t byte = codes[(int64_t)t * (len / 2) + (i >> 1)];
  const uint32_t code = (i & 1) ? (byte >> 4) : (byte & 0xF);
  const uint32_t mag = code & 7u;
  const float e2m1 = mag < 4 ? 0.5f * (float)mag : (mag == 4 ? 2.0f : mag == 5 ? 3.0f : mag == 6 ? 4.0f : 6.0f);
  const float s = e4m3_value(scales[scale_offset(t, i >> 4, len / 64)]);
  const float v = e2m1 * s * g;
  return (code & 8u) ? -v : v;
}

struct FactorView {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* g;
  int64_t len;
  int k;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Operands of the correction folded into the T_A GeMM (the second term of
// T_A^T = Q(B_R)^T Q(R_A) S_A + Q(R_B) S_B Z^T S_A, Z = Q(R_A)^T Q(L_B)):
//   blocks [0, zblocks):  FbZ (128 x fz_k; rows a < kA) = [Z S_B / alpha_TA hi | lo | 0],
//                         alpha_TA the T_A GeMM's tensor scales; a thread per (a, u)
//   blocks [zblocks, ..): FaZ rows = [Q(R_B) | Q(R_B) | 0] (bf16, exact), and the same two
//                         copies of Q(R_B) into the main fold operand Fb at [2 kpA, 2 kpA + 2 kpB)
// Z arrives as zsplits split-K partials of 128 x kpB, summed in order.  FbZ / FaZ are null
// when A has no factors (no correction, zblocks = 0).
constexpr int kRowsPerBlock = 32;
__global__ void __launch_bounds__(256) zfold_kernel(const float* __restrict__ Zp, int zsplits, int zblocks, int kA,
                                                    int kB, int kpA, int kpB, const float* __restrict__ SB,
                                                    const float* gBres, const float* gRA, FactorView RB, int fz_k,
                                                    __nv_bfloat16* __restrict__ FbZ, __nv_bfloat16* __restrict__ FaZ,
                                                    __nv_bfloat16* __restrict__ Fb, int fold_k, int64_t q) {
  if ((int)blockIdx.x < zblocks) {
    const int t = blockIdx.x * 256 + threadIdx.x;
    if (t >= 128 * kpB) return;
    const int a = t / kpB, u = t - (t / kpB) * kpB;
    float hi = 0.0f, lo = 0.0f;
    if (a < kA && u < kB) {
      const float inv_alpha = 1.0f / ((*gBres) * (*gRA));   // exact: powers of two
      float z = 0.0f;
      for (int s = 0; s < zsplits; ++s) z += Zp[((int64_t)s * 128 + a) * kpB + u];
      const float v = z * SB[u] * inv_alpha;
      hi = __bfloat162float(__float2bfloat16_rn(v));
      lo = v - hi;
    }
    FbZ[a * fz_k + u] = __float2bfloat16_rn(hi);
    FbZ[a * fz_k + kpB + u] = __float2bfloat16_rn(lo);
    for (int c = 2 * kpB + u; c < fz_k; c += kpB) FbZ[a * fz_k + c] = __float2bfloat16_rn(0.0f);
    return;
  }
  const int64_t i0 = (int64_t)(blockIdx.x - zblocks) * kRowsPerBlock;
  const float g = *RB.g;
  for (int e = threadIdx.x; e < kRowsPerBlock * kpB; e += blockDim.x) {
    const int r = e / kpB, u = e - (e / kpB) * kpB;
    const int64_t i = i0 + r;
    if (i >= q) continue;
    const __nv_bfloat16 v = __float2bfloat16_rn(u < kB ? factor_value(RB.codes, RB.scales, g, RB.len, u, i) : 0.0f);
    Fb[i * fold_k + 2 * kpA + u] = v;
    Fb[i * fold_k + 2 * kpA + kpB + u] = v;
    if (FaZ) {
      FaZ[i * fz_k + u] = v;
      FaZ[i * fz_k + kpB + u] = v;
      for (int c = 2 * kpB + u; c < fz_k; c += kpB) FaZ[i * fz_k + c] = __float2bfloat16_rn(0.0f);
    }
  }
}

// The main GeMM's fold operands, one warp per output row:
//   Fa rows i < p:  [Q(L_A) | Q(L_A) | T_B hi | T_B lo | 0] / alpha,  T_B = (sum of splits) S_B
//   Fb rows i < q:  [T_A^T hi | T_A^T lo | (Q(R_B) copies, written by zfold_kernel) | 0],
//                   T_A^T = (sum of splits) S_A
// alpha = gA * gB, the tensor scales of the main FP4 GeMM.  A lane owns columns j and j + 1
// of a kp-wide part and writes both of its copies (hi and lo, or the two Q(L_A) copies).
__global__ void __launch_bounds__(256) assemble_kernel(const float* __restrict__ TB, int bsplits, int64_t tb_stride,
                                                       const float* __restrict__ TA, int asplits, int64_t ta_stride,
                                                       const float* __restrict__ SA, const float* __restrict__ SB,
                                                       int kA, int kB, int kpA, int kpB, FactorView LA, int64_t p,
                                                       int64_t q, int fold_k, const float* ga, const float* gb,
                                                       __nv_bfloat16* __restrict__ Fa, __nv_bfloat16* __restrict__ Fb) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p + q) return;
  const bool is_a = row < p;
  const int64_t i = is_a ? row : row - p;
  __nv_bfloat16* dst = (is_a ? Fa : Fb) + i * fold_k;
  const float inv_alpha = is_a ? 1.0f / ((*ga) * (*gb)) : 1.0f;   // exact: a power of two
  // part 1 (columns [0, 2 kpA)): Q(L_A) copies on Fa rows, T_A^T hi / lo on Fb rows
  for (int j = 2 * lane; j < kpA; j += 64) {
    float v0 = 0.0f, v1 = 0.0f;
    if (is_a) {
      const float gl = *LA.g;
      if (j < kA) v0 = factor_value(LA.codes, LA.scales, gl, LA.len, j, i) * inv_alpha;
      if (j + 1 < kA) v1 = factor_value(LA.codes, LA.scales, gl, LA.len, j + 1, i) * inv_alpha;
      const uint32_t w = pack_bf16x2(v0, v1);
      *reinterpret_cast<uint32_t*>(dst + j) = w;
      *reinterpret_cast<uint32_t*>(dst + kpA + j) = w;
    } else {
      for (int s = 0; s < asplits; ++s) {
        const float2 t = *reinterpret_cast<const float2*>(TA + s * ta_stride + i * kpA + j);
        v0 += t.x;
        v1 += t.y;
      }
      v0 = j < kA ? v0 * SA[j] : 0.0f;
      v1 = j + 1 < kA ? v1 * SA[j + 1] : 0.0f;
      const float h0 = __bfloat162float(__float2bfloat16_rn(v0)), h1 = __bfloat162float(__float2bfloat16_rn(v1));
      *reinterpret_cast<uint32_t*>(dst + j) = pack_bf16x2(h0, h1);
      *reinterpret_cast<uint32_t*>(dst + kpA + j) = pack_bf16x2(v0 - h0, v1 - h1);
    }
  }
  // part 2 (columns [2 kpA, 2 kpA + 2 kpB)): T_B hi / lo on Fa rows (zfold_kernel fills Fb's)
  if (is_a) {
    for (int j = 2 * lane; j < kpB; j += 64) {
      float v0 = 0.0f, v1 = 0.0f;
      for (int s = 0; s < bsplits; ++s) {
        const float2 t = *reinterpret_cast<const float2*>(TB + s * tb_stride + i * kpB + j);
        v0 += t.x;
        v1 += t.y;
      }
      v0 = j < kB ? v0 * SB[j] * inv_alpha : 0.0f;
      v1 = j + 1 < kB ? v1 * SB[j + 1] * inv_alpha : 0.0f;
      const float h0 = __bfloat162float(__float2bfloat16_rn(v0)), h1 = __bfloat162float(__float2bfloat16_rn(v1));
      *reinterpret_cast<uint32_t*>(dst + 2 * kpA + j) = pack_bf16x2(h0, h1);
      *reinterpret_cast<uint32_t*>(dst + 2 * kpA + kpB + j) = pack_bf16x2(v0 - h0, v1 - h1);
    }
  }
  // padding columns
  for (int c = 2 * kpA + 2 * kpB + 2 * lane; c < fold_k; c += 64)
    *reinterpret_cast<uint32_t*>(dst + c) = 0u;
}

int pad_rank(int k) { return k == 0 ? 0 : k <= 16 ? 16 : k <= 32 ? 32 : 64; }

}  // namespace

metis_status check_factors(metis_ctx* ctx, const metis_factors* f, int64_t rows, int64_t cols);

metis_status run_linear(metis_ctx* ctx, const metis_operand* A, const metis_nvfp4* A_res, const metis_operand* B,
                        const metis_nvfp4* B_res, bool a_t, bool b_t, void* C, int64_t ldc, int32_t c_dtype) {
  const int64_t p = A_res->outer, K = A_res->inner, q = B_res->outer;
  if (B_res->inner != K) return fail(ctx, METIS_ERR_SHAPE, "operands disagree on the contraction length");
  if (c_dtype != METIS_OUT_F32 && c_dtype != METIS_OUT_BF16) return fail(ctx, METIS_ERR_ARG, "bad output dtype");
  if (ldc < q || ldc % (c_dtype == METIS_OUT_F32 ? 4 : 8)) return fail(ctx, METIS_ERR_ALIGN, "bad output leading dimension");
  // factor roles (see the header comment): A = U S V^T or its transpose, likewise B
  const metis_factors* fa = A->f;
  const metis_factors* fb = B->f;
  const int kA = fa ? fa->k : 0, kB = fb ? fb->k : 0;
  metis_status s;
  if (fa && kA > 0) {
    if ((s = check_factors(ctx, fa, a_t ? K : p, a_t ? p : K)) != METIS_OK) return s;
  }
  if (fb && kB > 0) {
    if ((s = check_factors(ctx, fb, b_t ? q : K, b_t ? K : q)) != METIS_OK) return s;
  }
  const metis_nvfp4* LAq = kA ? (a_t ? &fa->Vq : &fa->Uq) : nullptr;
  const metis_nvfp4* RAq = kA ? (a_t ? &fa->Uq : &fa->Vq) : nullptr;
  const metis_nvfp4* LBq = kB ? (b_t ? &fb->Vq : &fb->Uq) : nullptr;
  const metis_nvfp4* RBq = kB ? (b_t ? &fb->Uq : &fb->Vq) : nullptr;
  const int kpA = pad_rank(kA), kpB = pad_rank(kB);
  const int fold_k = (kA || kB) ? ((2 * kpA + 2 * kpB + 63) / 64) * 64 : 0;

  if (fold_k == 0) {
    GemmArgs g{A_res, B_res, nullptr, nullptr, 0, nullptr, C, ldc, c_dtype, 1.0f, q, 1, 0};
    return launch_gemm_nvfp4(ctx, g);
  }

  const bool corr = kA && kB;   // T_A picks up the correction Q(R_B) S_B Z^T S_A
  const int stagesK = (int)(K / 256);
  const int fz_k = corr ? ((2 * kpB + 63) / 64) * 64 : 0;
  const int zsplits = corr ? fp4_splits(ctx, 1, stagesK) : 0;
  const int bsplits = kB ? fp4_splits(ctx, p / 128, stagesK) : 0;
  const int asplits = kA ? fp4_splits(ctx, q / 128, stagesK + fz_k / 64) : 0;
  const size_t need = 256 * 12 + (size_t)bsplits * p * kpB * 4 + (size_t)asplits * q * kpA * 4 +
                      (size_t)zsplits * 128 * kpB * 4 + (size_t)q * fz_k * 2 + (size_t)128 * fz_k * 2 +
                      (size_t)p * fold_k * 2 + (size_t)q * fold_k * 2;
  if ((s = ensure_workspace(ctx, need)) != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  float* TB32 = static_cast<float*>(ws.take((size_t)std::max(bsplits, 1) * p * std::max(kpB, 1) * 4));
  float* TA32 = static_cast<float*>(ws.take((size_t)std::max(asplits, 1) * q * std::max(kpA, 1) * 4));
  float* Zp = static_cast<float*>(ws.take((size_t)std::max(zsplits, 1) * 128 * std::max(kpB, 1) * 4));
  __nv_bfloat16* FaZ = static_cast<__nv_bfloat16*>(ws.take((size_t)q * std::max(fz_k, 64) * 2));
  __nv_bfloat16* FbZ = static_cast<__nv_bfloat16*>(ws.take((size_t)128 * std::max(fz_k, 64) * 2));
  __nv_bfloat16* Fa = static_cast<__nv_bfloat16*>(ws.take((size_t)p * fold_k * 2));
  __nv_bfloat16* Fb = static_cast<__nv_bfloat16*>(ws.take((size_t)q * fold_k * 2));
  if (!Fb) return fail(ctx, METIS_ERR_WORKSPACE, "fold workspace layout");
  cudaStream_t st = ctx->stream;

  FactorView vLA{}, vRB{};
  if (kA) vLA = {LAq->codes, LAq->scales, LAq->tensor_scale, LAq->inner, kA};
  if (kB) vRB = {RBq->codes, RBq->scales, RBq->tensor_scale, RBq->inner, kB};
  // Z = Q(R_A)^T Q(L_B) on the tensor cores (128 x kpB, split-K over the contraction length)
  if (corr) {
    GemmArgs g{RAq, LBq, nullptr, nullptr, 0, nullptr, Zp, kpB, METIS_OUT_F32, 1.0f, kpB, zsplits, 128 * kpB};
    if ((s = launch_gemm_nvfp4(ctx, g)) != METIS_OK) return s;
  }
  if (kB) {
    const int zblocks = corr ? (128 * kpB + 255) / 256 : 0;
    zfold_kernel<<<(unsigned)(zblocks + (q + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, st>>>(
        Zp, zsplits, zblocks, kA, kB, kpA, kpB, fb->S, B_res->tensor_scale, corr ? RAq->tensor_scale : nullptr,
        vRB, fz_k, corr ? FbZ : nullptr, corr ? FaZ : nullptr, Fb, fold_k, q); count_launch();
    // T_B = Q(A_R) Q(L_B)  (p x kpB partials; S_B applied when assembling)
    GemmArgs g{A_res, LBq, nullptr, nullptr, 0, nullptr, TB32, kpB, METIS_OUT_F32, 1.0f, kpB, bsplits,
               p * kpB};
    if ((s = launch_gemm_nvfp4(ctx, g)) != METIS_OK) return s;
  }
  // T_A^T / S_A = Q(B_R)^T Q(R_A) + [Q(R_B) | Q(R_B)] [Z S_B hi | lo]^T / alpha_TA  (q x kpA partials)
  if (kA) {
    GemmArgs g{B_res, RAq, corr ? FaZ : nullptr, corr ? FbZ : nullptr, fz_k, nullptr, TA32, kpA, METIS_OUT_F32,
               1.0f, kpA, asplits, q * kpA};
    if ((s = launch_gemm_nvfp4(ctx, g)) != METIS_OK) return s;
  }
  assemble_kernel<<<(unsigned)((p + q + 7) / 8), 256, 0, st>>>(TB32, bsplits, p * kpB, TA32, asplits, q * kpA,
                                                               kA ? fa->S : nullptr, kB ? fb->S : nullptr, kA, kB,
                                                               kpA, kpB, vLA, p, q, fold_k, A_res->tensor_scale,
                                                               B_res->tensor_scale, Fa, Fb); count_launch();
  if ((s = check_cuda(ctx, cudaGetLastError(), "fold preparation")) != METIS_OK) return s;
  GemmArgs g{A_res, B_res, Fa, Fb, fold_k, nullptr, C, ldc, c_dtype, 1.0f, q, 1, 0};
  return launch_gemm_nvfp4(ctx, g);
}

}  // namespace metis
