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

// Decoded value of a k x len factor NVFP4 tensor (the transposed storage of a len x k
// factor) at row t, column r0 + r, from a block's staged copy of columns r0 .. r0 + 31:
// 16 code bytes and 2 block scales per row t.
__device__ __forceinline__ float staged_factor(const uint8_t* fcodes, const uint8_t* fscales, float g, int t, int r) {
  const uint8_t byte = fcodes[t * 16 + (r >> 1)];
  const uint32_t code = (r & 1) ? (byte >> 4) : (byte & 0xF);
  const uint32_t mag = code & 7u;
  const float e2m1 = mag < 4 ? 0.5f * (float)mag : (mag == 4 ? 2.0f : mag == 5 ? 3.0f : mag == 6 ? 4.0f : 6.0f);
  const float v = e2m1 * e4m3_value(fscales[t * 2 + (r >> 4)]) * g;
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

// a + the sum over sp < n of the float pairs at base + sp * stride, taken in split order;
// the loads go out four at a time
__device__ __forceinline__ float2 add_splits(float2 a, const float* base, int64_t stride, int n) {
  for (int s0 = 0; s0 < n; s0 += 4) {
    float2 t[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      t[u] = s0 + u < n ? *reinterpret_cast<const float2*>(base + (s0 + u) * stride) : make_float2(0.0f, 0.0f);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < n) {
        a.x += t[u].x;
        a.y += t[u].y;
      }
  }
  return a;
}

// The main GeMM's fold operands, 32 rows per block (8 warps, 4 consecutive rows each,
// formed together; a lane owns columns j and j + 1 of a kp-wide part and writes both of
// its copies):
//   Fa rows i < p:  [Q(L_A) | Q(L_A) | T_B hi | T_B lo | 0] / alpha,
//                   T_B = (sum of the splits of Q(A_R) Q(L_B)) S_B
//   Fb rows i < q:  [T_A^T hi | T_A^T lo | Q(R_B) | Q(R_B) | 0],
//                   T_A^T = (sum of the splits of Q(B_R)^T Q(R_A) + Q(R_B) S_B Z^T) S_A,
//                   Z = Q(R_A)^T Q(L_B) (sum of its splits)
// alpha = gA * gB, the tensor scales of the main FP4 GeMM.  The correction Q(R_B) S_B Z^T
// (k_B terms per entry) is formed here in fp32: a block of Fb rows first stages
// S_B[u] Z[a][u] in shared memory (u-major, so the lanes read consecutive a).
constexpr int kFoldRows = 32;
__global__ void __launch_bounds__(256) fold_assemble_kernel(
    const float* __restrict__ TB, int bsplits, int64_t tb_stride, const float* __restrict__ TA, int asplits,
    int64_t ta_stride, const float* __restrict__ Zp, int zsplits, const float* __restrict__ SA,
    const float* __restrict__ SB, int kA, int kB, int kpA, int kpB, FactorView LA, FactorView RB, int64_t p, int64_t q,
    int fold_k, const float* ga, const float* gb, __nv_bfloat16* __restrict__ Fa, __nv_bfloat16* __restrict__ Fb) {
  __shared__ float zs[64 * 66];   // zs[u * 66 + a] = S_B[u] Z[a][u] (row pitch 66: fewer bank conflicts)
  __shared__ __align__(16) float rbs[8][64 * 4];   // per warp: Q(R_B)(i, u) of the warp's 4 rows, u-major
  // the block's 32 rows of the factor it decodes (Q(L_A) on Fa rows, Q(R_B) on Fb rows):
  // 16 code bytes and 2 scale bytes per factor column t, staged with coalesced loads
  __shared__ uint8_t fcodes[64 * 16];
  __shared__ uint8_t fscales[64 * 2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nbA = (p + kFoldRows - 1) / kFoldRows;
  const bool is_a = (int64_t)blockIdx.x < nbA;
  const int64_t r0 = (is_a ? (int64_t)blockIdx.x : (int64_t)blockIdx.x - nbA) * kFoldRows;
  const bool corr = !is_a && Zp != nullptr;
  if (corr) {
    // thread (u = tid mod 64, a = tid / 64 + 4 t): a warp reads 32 consecutive u of one row
    // of Z; all 16 x zsplits loads of a thread are independent, so they overlap
    const int u = threadIdx.x & 63, a0 = threadIdx.x >> 6;
    float z[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) z[t] = 0.0f;
    if (u < kB) {
      for (int sp = 0; sp < zsplits; ++sp) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int a = a0 + 4 * t;
          if (a < kA) z[t] += Zp[((int64_t)sp * 128 + a) * kpB + u];
        }
      }
    }
    const float sb = u < kB ? SB[u] : 0.0f;
#pragma unroll
    for (int t = 0; t < 16; ++t) zs[u * 66 + a0 + 4 * t] = sb * z[t];
    __syncthreads();
  }
  {
    const FactorView& F = is_a ? LA : RB;
    const int kF = is_a ? kA : kB;
    for (int e = threadIdx.x; e < kF * 4; e += blockDim.x) {
      const int t = e >> 2, c = e & 3;
      *reinterpret_cast<uint32_t*>(fcodes + t * 16 + c * 4) =
          *reinterpret_cast<const uint32_t*>(F.codes + (int64_t)t * (F.len / 2) + r0 / 2 + c * 4);
    }
    for (int e = threadIdx.x; e < kF * 2; e += blockDim.x) {
      const int t = e >> 1, b = e & 1;
      fscales[t * 2 + b] = F.scales[scale_offset(t, (r0 >> 4) + b, F.len / 64)];
    }
    __syncthreads();
  }
  const float inv_alpha = is_a ? 1.0f / ((*ga) * (*gb)) : 1.0f;   // exact: a power of two
  // a warp owns 4 consecutive rows and forms them together, so that the split partials of
  // its rows are loaded together and every shared-memory value feeds four rows
  constexpr int kRowsPerWarp = kFoldRows / 8;
  const int rr0 = warp * kRowsPerWarp;
  const int64_t nrows = is_a ? p : q;
  bool live[kRowsPerWarp];
  __nv_bfloat16* dst[kRowsPerWarp];
#pragma unroll
  for (int x = 0; x < kRowsPerWarp; ++x) {
    live[x] = r0 + rr0 + x < nrows;
    dst[x] = (is_a ? Fa : Fb) + (r0 + rr0 + x) * fold_k;
  }
  if (is_a) {
    // Q(L_A) copies
    const float gl = kA ? *LA.g : 1.0f;
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      if (!live[x]) continue;
      for (int j = 2 * lane; j < kpA; j += 64) {
        const float v0 = j < kA ? staged_factor(fcodes, fscales, gl, j, rr0 + x) * inv_alpha : 0.0f;
        const float v1 = j + 1 < kA ? staged_factor(fcodes, fscales, gl, j + 1, rr0 + x) * inv_alpha : 0.0f;
        const uint32_t w = pack_bf16x2(v0, v1);
        *reinterpret_cast<uint32_t*>(dst[x] + j) = w;
        *reinterpret_cast<uint32_t*>(dst[x] + kpA + j) = w;
      }
    }
    // T_B hi / lo
    for (int j = 2 * lane; j < kpB; j += 64) {
      float2 a[kRowsPerWarp];
#pragma unroll
      for (int x = 0; x < kRowsPerWarp; ++x) a[x] = make_float2(0.0f, 0.0f);
      for (int sp = 0; sp < bsplits; ++sp) {
        float2 t[kRowsPerWarp];
#pragma unroll
        for (int x = 0; x < kRowsPerWarp; ++x)
          t[x] = live[x] ? *reinterpret_cast<const float2*>(TB + sp * tb_stride + (r0 + rr0 + x) * kpB + j)
                         : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int x = 0; x < kRowsPerWarp; ++x) {
          a[x].x += t[x].x;
          a[x].y += t[x].y;
        }
      }
#pragma unroll
      for (int x = 0; x < kRowsPerWarp; ++x) {
        if (!live[x]) continue;
        const float v0 = j < kB ? a[x].x * SB[j] * inv_alpha : 0.0f;
        const float v1 = j + 1 < kB ? a[x].y * SB[j + 1] * inv_alpha : 0.0f;
        const float h0 = __bfloat162float(__float2bfloat16_rn(v0)), h1 = __bfloat162float(__float2bfloat16_rn(v1));
        *reinterpret_cast<uint32_t*>(dst[x] + 2 * kpA + j) = pack_bf16x2(h0, h1);
        *reinterpret_cast<uint32_t*>(dst[x] + 2 * kpA + kpB + j) = pack_bf16x2(v0 - h0, v1 - h1);
      }
    }
  } else {
    // Q(R_B)(i, u) for u = lane and lane + 32 (exact in bf16), staged u-major for the
    // correction: rbs[warp][u][x]
    const float gr = kB ? *RB.g : 1.0f;
    float rb[kRowsPerWarp][2];
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      rb[x][0] = lane < kB ? staged_factor(fcodes, fscales, gr, lane, rr0 + x) : 0.0f;
      rb[x][1] = lane + 32 < kB ? staged_factor(fcodes, fscales, gr, lane + 32, rr0 + x) : 0.0f;
    }
    // T_A^T hi / lo: lane owns columns j, j + 1 (kpA <= 64, so at most one pair per lane)
    const int j = 2 * lane;
    float2 c[kRowsPerWarp];
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) c[x] = make_float2(0.0f, 0.0f);
    if (corr) {
      *reinterpret_cast<float4*>(&rbs[warp][lane * 4]) = make_float4(rb[0][0], rb[1][0], rb[2][0], rb[3][0]);
      *reinterpret_cast<float4*>(&rbs[warp][(lane + 32) * 4]) = make_float4(rb[0][1], rb[1][1], rb[2][1], rb[3][1]);
      __syncwarp();
      if (j < kpA) {
        // eight independent sums (4 rows x 2 columns) per lane, each over u in order
        for (int u = 0; u < kB; ++u) {
          const float4 r = *reinterpret_cast<const float4*>(&rbs[warp][u * 4]);
          const float2 z = *reinterpret_cast<const float2*>(zs + u * 66 + j);
          const float rv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int x = 0; x < kRowsPerWarp; ++x) {
            c[x].x = fmaf(rv[x], z.x, c[x].x);
            c[x].y = fmaf(rv[x], z.y, c[x].y);
          }
        }
      }
    }
    if (j < kpA) {
      for (int sp = 0; sp < asplits; ++sp) {
        float2 t[kRowsPerWarp];
#pragma unroll
        for (int x = 0; x < kRowsPerWarp; ++x)
          t[x] = live[x] ? *reinterpret_cast<const float2*>(TA + sp * ta_stride + (r0 + rr0 + x) * kpA + j)
                         : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int x = 0; x < kRowsPerWarp; ++x) {
          c[x].x += t[x].x;
          c[x].y += t[x].y;
        }
      }
#pragma unroll
      for (int x = 0; x < kRowsPerWarp; ++x) {
        if (!live[x]) continue;
        const float v0 = j < kA ? c[x].x * SA[j] : 0.0f;
        const float v1 = j + 1 < kA ? c[x].y * SA[j + 1] : 0.0f;
        const float h0 = __bfloat162float(__float2bfloat16_rn(v0)), h1 = __bfloat162float(__float2bfloat16_rn(v1));
        *reinterpret_cast<uint32_t*>(dst[x] + j) = pack_bf16x2(h0, h1);
        *reinterpret_cast<uint32_t*>(dst[x] + kpA + j) = pack_bf16x2(v0 - h0, v1 - h1);
      }
    }
    // Q(R_B) copies
#pragma unroll
    for (int x = 0; x < kRowsPerWarp; ++x) {
      if (!live[x]) continue;
      for (int u = lane; u < kpB; u += 32) {
        const __nv_bfloat16 v = __float2bfloat16_rn(u < 32 ? rb[x][0] : rb[x][1]);
        dst[x][2 * kpA + u] = v;
        dst[x][2 * kpA + kpB + u] = v;
      }
    }
  }
  // padding columns
#pragma unroll
  for (int x = 0; x < kRowsPerWarp; ++x) {
    if (!live[x]) continue;
    for (int cc = 2 * kpA + 2 * kpB + 2 * lane; cc < fold_k; cc += 64) *reinterpret_cast<uint32_t*>(dst[x] + cc) = 0u;
  }
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
  // one split count for the three thin GeMMs of one grouped launch (about two units per SM)
  const int64_t thin_tiles = (corr ? 1 : 0) + (kB ? p / 128 : 0) + (kA ? q / 128 : 0);
  const int splits = fp4_splits(ctx, thin_tiles, stagesK);
  const int zsplits = corr ? splits : 0, bsplits = kB ? splits : 0, asplits = kA ? splits : 0;
  const size_t need = 256 * 8 + (size_t)bsplits * p * kpB * 4 + (size_t)asplits * q * kpA * 4 +
                      (size_t)zsplits * 128 * kpB * 4 + (size_t)p * fold_k * 2 + (size_t)q * fold_k * 2;
  if ((s = ensure_workspace(ctx, need)) != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  float* TB32 = static_cast<float*>(ws.take((size_t)std::max(bsplits, 1) * p * std::max(kpB, 1) * 4));
  float* TA32 = static_cast<float*>(ws.take((size_t)std::max(asplits, 1) * q * std::max(kpA, 1) * 4));
  float* Zp = static_cast<float*>(ws.take((size_t)std::max(zsplits, 1) * 128 * std::max(kpB, 1) * 4));
  __nv_bfloat16* Fa = static_cast<__nv_bfloat16*>(ws.take((size_t)p * fold_k * 2));
  __nv_bfloat16* Fb = static_cast<__nv_bfloat16*>(ws.take((size_t)q * fold_k * 2));
  if (!Fb) return fail(ctx, METIS_ERR_WORKSPACE, "fold workspace layout");
  cudaStream_t st = ctx->stream;

  // the thin GeMMs: Z = Q(R_A)^T Q(L_B) (128 x kpB), T_B = Q(A_R) Q(L_B) (p x kpB) and
  // T_A^T / S_A = Q(B_R)^T Q(R_A) (q x kpA), as split-K fp32 partials, in one launch when
  // their widths agree
  GemmArgs thin[3];
  int nthin = 0;
  if (corr) thin[nthin++] = GemmArgs{RAq, LBq, nullptr, nullptr, 0, nullptr, Zp, kpB, METIS_OUT_F32, 1.0f, kpB,
                                     zsplits, 128 * kpB};
  if (kB) thin[nthin++] = GemmArgs{A_res, LBq, nullptr, nullptr, 0, nullptr, TB32, kpB, METIS_OUT_F32, 1.0f, kpB,
                                   bsplits, p * kpB};
  if (kA) thin[nthin++] = GemmArgs{B_res, RAq, nullptr, nullptr, 0, nullptr, TA32, kpA, METIS_OUT_F32, 1.0f, kpA,
                                   asplits, q * kpA};
  if (kpA == kpB || !kA || !kB) {
    if ((s = launch_gemm_nvfp4_group(ctx, thin, nthin)) != METIS_OK) return s;
  } else {
    for (int i = 0; i < nthin; ++i)
      if ((s = launch_gemm_nvfp4(ctx, thin[i])) != METIS_OK) return s;
  }
  FactorView vLA{}, vRB{};
  if (kA) vLA = {LAq->codes, LAq->scales, LAq->tensor_scale, LAq->inner, kA};
  if (kB) vRB = {RBq->codes, RBq->scales, RBq->tensor_scale, RBq->inner, kB};
  const int64_t blocks = (p + kFoldRows - 1) / kFoldRows + (q + kFoldRows - 1) / kFoldRows;
  fold_assemble_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      TB32, bsplits, p * kpB, TA32, asplits, q * kpA, corr ? Zp : nullptr, zsplits, kA ? fa->S : nullptr,
      kB ? fb->S : nullptr, kA, kB, kpA, kpB, vLA, vRB, p, q, fold_k, A_res->tensor_scale, B_res->tensor_scale, Fa,
      Fb);
  count_launch();
  if ((s = check_cuda(ctx, cudaGetLastError(), "fold preparation")) != METIS_OK) return s;
  GemmArgs g{A_res, B_res, Fa, Fb, fold_k, nullptr, C, ldc, c_dtype, 1.0f, q, 1, 0};
  return launch_gemm_nvfp4(ctx, g);
}

}  // namespace metis
