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

// Partial Z = Q(L)^T Q(R) over one chunk of the shared length (kL x kR).
constexpr int kZChunk = 64;
__global__ void z_partial_kernel(FactorView L, FactorView R, float* partial) {
  __shared__ float sl[64][kZChunk + 1];
  __shared__ float sr[64][kZChunk + 1];
  const int64_t i0 = (int64_t)blockIdx.x * kZChunk;
  const float gl = *L.g, gr = *R.g;
  for (int e = threadIdx.x; e < 64 * kZChunk; e += blockDim.x) {
    const int t = e / kZChunk, c = e % kZChunk;
    sl[t][c] = t < L.k ? factor_value(L.codes, L.scales, gl, L.len, t, i0 + c) : 0.0f;
    sr[t][c] = t < R.k ? factor_value(R.codes, R.scales, gr, R.len, t, i0 + c) : 0.0f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 64 * 64; e += blockDim.x) {
    const int a = e / 64, b = e % 64;
    float acc = 0.0f;
    if (a < L.k && b < R.k)
      for (int c = 0; c < kZChunk; ++c) acc = fmaf(sl[a][c], sr[b][c], acc);
    partial[(int64_t)blockIdx.x * 4096 + e] = acc;
  }
}

// Z[a][b] = sum over chunks in a fixed order (deterministic).
__global__ void z_reduce_kernel(const float* partial, int nchunks, float* Z) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 4096) return;
  float acc = 0.0f;
  for (int c = 0; c < nchunks; ++c) acc += partial[(int64_t)c * 4096 + e];
  Z[e] = acc;
}

// Fb rows: [T_A^T hi | T_A^T lo | Q(R_B) | Q(R_B)] with
// T_A^T[i][j] = TA32[i][j] + sum_u Q(R_B)[i][u] S_B[u] Z[j][u] S_A[j]   (Z = Q(R_A)^T Q(L_B)).
// One block per 32 rows: the decoded rows of Q(R_B) and the k x k correction
// C2[u][j] = S_B[u] Z[j][u] S_A[j] are staged once in shared memory.
constexpr int kFoldRows = 32;
__global__ void fold_b_kernel(const float* __restrict__ TA32, int kpA, int kA, FactorView RB, int kpB,
                              const float* __restrict__ SA, const float* __restrict__ SB, const float* __restrict__ Z,
                              int64_t q, int fold_k, __nv_bfloat16* __restrict__ Fb) {
  __shared__ float qrb[kFoldRows][65];
  __shared__ float c2[64][65];
  const int64_t i0 = (int64_t)blockIdx.x * kFoldRows;
  const float gr = RB.k > 0 ? *RB.g : 0.0f;
  for (int e = threadIdx.x; e < kFoldRows * 64; e += blockDim.x) {
    const int r = e / 64, u = e % 64;
    qrb[r][u] = (u < RB.k) ? factor_value(RB.codes, RB.scales, gr, RB.len, u, i0 + r) : 0.0f;
  }
  if (RB.k > 0 && kA > 0) {
    for (int e = threadIdx.x; e < 64 * 64; e += blockDim.x) {
      const int u = e / 64, j = e % 64;
      c2[u][j] = (u < RB.k && j < kA) ? SB[u] * Z[j * 64 + u] * SA[j] : 0.0f;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kFoldRows * fold_k; e += blockDim.x) {
    const int r = e / fold_k, c = e % fold_k;
    const int64_t i = i0 + r;
    float out = 0.0f;
    if (c < 2 * kpA) {
      const int j = c < kpA ? c : c - kpA;
      float t = 0.0f;
      if (j < kA) {
        t = TA32[i * kpA + j];
        if (RB.k > 0) {
          float acc = 0.0f;
          for (int u = 0; u < RB.k; ++u) acc = fmaf(qrb[r][u], c2[u][j], acc);
          t += acc;
        }
      }
      const __nv_bfloat16 hi = __float2bfloat16_rn(t);
      out = c < kpA ? __bfloat162float(hi) : t - __bfloat162float(hi);
    } else if (c < 2 * kpA + 2 * kpB) {
      out = qrb[r][(c - 2 * kpA) % kpB];
    }
    Fb[i * fold_k + c] = __float2bfloat16_rn(out);
  }
}

// Fa rows: [Q(L_A) | Q(L_A) | T_B hi | T_B lo] / alpha.
__global__ void fold_a_kernel(const float* __restrict__ TB32, int kpB, int kB, FactorView LA, int kpA, int64_t p,
                              int fold_k, const float* ga, const float* gb, __nv_bfloat16* __restrict__ Fa) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p * fold_k) return;
  const int64_t i = idx / fold_k;
  const int c = (int)(idx - i * fold_k);
  const float inv_alpha = 1.0f / ((*ga) * (*gb));  // exact: a power of two
  float out = 0.0f;
  if (c < 2 * kpA) {
    const int u = c % kpA;
    out = u < LA.k ? factor_value(LA.codes, LA.scales, *LA.g, LA.len, u, i) * inv_alpha : 0.0f;
  } else if (c < 2 * kpA + 2 * kpB) {
    const int j = (c - 2 * kpA) % kpB;
    const float t = j < kB ? TB32[i * kpB + j] * inv_alpha : 0.0f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(t);
    out = (c - 2 * kpA) < kpB ? __bfloat162float(hi) : t - __bfloat162float(hi);
  }
  Fa[i * fold_k + c] = __float2bfloat16_rn(out);
}

__global__ void pad_sigma_kernel(const float* S, int k, int kp, float* out) {
  const int i = threadIdx.x;
  if (i < kp) out[i] = i < k ? S[i] : 0.0f;
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
    GemmArgs g{A_res, B_res, nullptr, nullptr, 0, nullptr, C, ldc, c_dtype, 1.0f, q};
    return launch_gemm_nvfp4(ctx, g);
  }

  const int nchunks = (int)(K / kZChunk);
  const size_t need = 256 * 12 + (size_t)p * kpB * 4 + (size_t)q * kpA * 4 + (size_t)nchunks * 4096 * 4 + 4096 * 4 +
                      2 * 64 * 4 + (size_t)p * fold_k * 2 + (size_t)q * fold_k * 2;
  if ((s = ensure_workspace(ctx, need)) != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  float* TB32 = static_cast<float*>(ws.take((size_t)p * std::max(kpB, 1) * 4));
  float* TA32 = static_cast<float*>(ws.take((size_t)q * std::max(kpA, 1) * 4));
  float* Zp = static_cast<float*>(ws.take((size_t)nchunks * 4096 * 4));
  float* Z = static_cast<float*>(ws.take(4096 * 4));
  float* SAp = static_cast<float*>(ws.take(64 * 4));
  float* SBp = static_cast<float*>(ws.take(64 * 4));
  __nv_bfloat16* Fa = static_cast<__nv_bfloat16*>(ws.take((size_t)p * fold_k * 2));
  __nv_bfloat16* Fb = static_cast<__nv_bfloat16*>(ws.take((size_t)q * fold_k * 2));
  cudaStream_t st = ctx->stream;

  FactorView vLA{}, vRA{}, vLB{}, vRB{};
  if (kA) {
    vLA = {LAq->codes, LAq->scales, LAq->tensor_scale, LAq->inner, kA};
    vRA = {RAq->codes, RAq->scales, RAq->tensor_scale, RAq->inner, kA};
    pad_sigma_kernel<<<1, 64, 0, st>>>(fa->S, kA, kpA, SAp); count_launch();
  }
  if (kB) {
    vLB = {LBq->codes, LBq->scales, LBq->tensor_scale, LBq->inner, kB};
    vRB = {RBq->codes, RBq->scales, RBq->tensor_scale, RBq->inner, kB};
    pad_sigma_kernel<<<1, 64, 0, st>>>(fb->S, kB, kpB, SBp); count_launch();
  }
  // T_B = Q(A_R) Q(L_B) S_B  (p x kpB, fp32)
  if (kB) {
    GemmArgs g{A_res, LBq, nullptr, nullptr, 0, SBp, TB32, kpB, METIS_OUT_F32, 1.0f, kpB};
    if ((s = launch_gemm_nvfp4(ctx, g)) != METIS_OK) return s;
  }
  // first part of T_A^T = Q(B_R)^T Q(R_A) S_A  (q x kpA, fp32)
  if (kA) {
    GemmArgs g{B_res, RAq, nullptr, nullptr, 0, SAp, TA32, kpA, METIS_OUT_F32, 1.0f, kpA};
    if ((s = launch_gemm_nvfp4(ctx, g)) != METIS_OK) return s;
  }
  // Z = Q(R_A)^T Q(L_B)  (kA x kB over the contraction length K)
  if (kA && kB) {
    z_partial_kernel<<<nchunks, 256, 0, st>>>(vRA, vLB, Zp); count_launch();
    z_reduce_kernel<<<16, 256, 0, st>>>(Zp, nchunks, Z); count_launch();
  }
  if (kA || kB) {
    fold_b_kernel<<<(unsigned)(q / kFoldRows), 256, 0, st>>>(TA32, kpA, kA, vRB, kpB, SAp, SBp, Z, q, fold_k,
                                                             Fb); count_launch();
    fold_a_kernel<<<(unsigned)((p * fold_k + 255) / 256), 256, 0, st>>>(TB32, kpB, kB, vLA, kpA, p, fold_k,
                                                                        A_res->tensor_scale, B_res->tensor_scale, Fa); count_launch();
  }
  if ((s = check_cuda(ctx, cudaGetLastError(), "fold preparation")) != METIS_OK) return s;
  GemmArgs g{A_res, B_res, Fa, Fb, fold_k, nullptr, C, ldc, c_dtype, 1.0f, q};
  return launch_gemm_nvfp4(ctx, g);
}

}  // namespace metis
