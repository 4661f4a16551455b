// The LoRA-SVD linear projection on the library's kernels.
//
// Method: "Full-Stack FP4: stable LLM pretraining with quantized projections, optimizer
// and attention" (gist.science technical summary), section 2.1 (LoRA-SVD linear
// projection).  The weight is parameterized as
//     W = W_res + beta L2 L1          (L2: m x k, L1: k x n)
// with the compact principal subspace L2 L1 kept in high precision (bf16 on the tensor
// cores, fp32 masters) and the residual W_res computed in NVFP4.  Updates of L2 are kept
// in the subspace by a Cholesky-QR constraint, and every so many steps the split is
// realigned by a randomized SVD of W.
//
// The products are evaluated with the Metis kernels:
//   forward        Y  = Q(X) Q(W_res) + beta (X L2) L1
//   input gradient dX = Q(D) Q(W_res)^T + beta (D L1^T) L2^T
// each as ONE fused FP4 GeMM whose bf16 rank fold carries the branch:
//   Fa = [beta T hi | beta T lo] / alpha,  Fb = [Lout | Lout],  T = M Lin (fp32, tensor
//   cores), alpha = gA gB the tensor-scale product the fused kernel multiplies by;
//   branch gradients  dL2 = beta X^T (D L1^T),  dL1^T = beta D^T (X L2)  on the bf16
//   tensor cores from M^T and T;
//   constraint        L2 = Q R (CholQR), L2 <- Q, L1 <- R L1  (the product is unchanged);
//   realignment       W_eff = W_res + beta L2 L1 = U S V^T + ...  (randomized SVD, rank k),
//                     L2 <- U, L1 <- S V^T / beta, W_res <- W_eff - beta L2 L1.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace metis {
namespace {

constexpr int kLoraRows = 32;   // rows of Fa / Fb per block of the fold kernel

unsigned blocks_of(int64_t n, int t = 256) { return (unsigned)((n + t - 1) / t); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// out (kp x K bf16, K-major) = bf16(Lin)^T, rows k .. kp - 1 zero.  Lin(x, j) is
// L[x * k + j] (a K x k factor, as L2 in the forward) or L[j * K + x] (a k x K factor,
// as L1 in the input gradient).
__global__ void lora_pack_in_kernel(const float* __restrict__ L, bool k_major, int64_t K, int k, int kp,
                                    __nv_bfloat16* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)kp * K) return;
  const int j = (int)(e / K);
  const int64_t x = e - (int64_t)j * K;
  float v = 0.0f;
  if (j < k) v = k_major ? L[(int64_t)j * K + x] : L[x * k + j];
  out[e] = __float2bfloat16_rn(v);
}

// Fold operands of the branch.  Blocks [0, p / 32) write 32 rows of Fa each:
//   Fa[i] = [v hi | v lo | 0 ...],  v = beta * T[i] / alpha,  T[i][j] = sum over the
//   split partials (in order) of M Lin, and T itself (fp32, p x k) when T_out is given;
// the remaining blocks write 32 rows of Fb each: Fb[c] = [Lout(c, :) | Lout(c, :) | 0 ...]
// in bf16, Lout(c, j) = L1[j * q + c] (forward) or L2[c * k + j] (input gradient).
__global__ void __launch_bounds__(256) lora_fold_kernel(const float* __restrict__ Tp, int splits, int64_t p, int k,
                                                        int kp, float beta, const float* ga, const float* gb,
                                                        const float* __restrict__ Lout, bool lout_k_major, int64_t q,
                                                        int fold_k, float* __restrict__ T_out,
                                                        __nv_bfloat16* __restrict__ Fa,
                                                        __nv_bfloat16* __restrict__ Fb) {
  __shared__ float lo_s[kLoraRows][65];
  const int64_t nbA = p / kLoraRows;
  const int half = fold_k / 2;   // bf16 pairs per row
  if ((int64_t)blockIdx.x < nbA) {
    const int64_t r0 = (int64_t)blockIdx.x * kLoraRows;
    const float scale = beta / ((*ga) * (*gb));   // dividing by alpha is exact: a power of two
    const int64_t stride = p * kp;
    for (int e = threadIdx.x; e < kLoraRows * half; e += blockDim.x) {
      const int rr = e / half, j = 2 * (e - (e / half) * half);
      const int64_t i = r0 + rr;
      uint32_t word = 0u;
      if (j < 2 * kp) {
        const int jj = j < kp ? j : j - kp;
        float t0 = 0.0f, t1 = 0.0f;
        for (int sp = 0; sp < splits; ++sp) {
          const float2 t = *reinterpret_cast<const float2*>(Tp + sp * stride + i * kp + jj);
          t0 += t.x;
          t1 += t.y;
        }
        const float v0 = t0 * scale, v1 = t1 * scale;
        const float h0 = __bfloat162float(__float2bfloat16_rn(v0)), h1 = __bfloat162float(__float2bfloat16_rn(v1));
        if (j < kp) {
          word = pack2(h0, h1);
          if (T_out) {
            if (jj < k) T_out[i * k + jj] = t0;
            if (jj + 1 < k) T_out[i * k + jj + 1] = t1;
          }
        } else {
          word = pack2(v0 - h0, v1 - h1);
        }
      }
      *reinterpret_cast<uint32_t*>(Fa + i * fold_k + j) = word;
    }
  } else {
    const int64_t c0 = ((int64_t)blockIdx.x - nbA) * kLoraRows;
    for (int e = threadIdx.x; e < kLoraRows * k; e += blockDim.x) {
      if (lout_k_major) {
        const int j = e / kLoraRows, cc = e - (e / kLoraRows) * kLoraRows;
        lo_s[cc][j] = Lout[(int64_t)j * q + c0 + cc];
      } else {
        const int cc = e / k, j = e - (e / k) * k;
        lo_s[cc][j] = Lout[(c0 + cc) * k + j];
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kLoraRows * half; e += blockDim.x) {
      const int cc = e / half, j = 2 * (e - (e / half) * half);
      float v0 = 0.0f, v1 = 0.0f;
      if (j < 2 * kp) {
        const int jj = j < kp ? j : j - kp;
        if (jj < k) v0 = lo_s[cc][jj];
        if (jj + 1 < k) v1 = lo_s[cc][jj + 1];
      }
      *reinterpret_cast<uint32_t*>(Fb + (c0 + cc) * fold_k + j) = pack2(v0, v1);
    }
  }
}

// G = beta * (sum over splits, in order, of the hi and lo halves of the partials):
// G[i * k + j] (c x k) or, transposed, G[j * c + i] (k x c).
__global__ void lora_grad_reduce_kernel(const float* __restrict__ partial, int splits, int64_t c, int kp, int k,
                                        float beta, bool transpose_out, float* __restrict__ G) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= c * k) return;
  int64_t i;
  int j;
  if (transpose_out) {
    j = (int)(e / c);
    i = e - (int64_t)j * c;
  } else {
    i = e / k;
    j = (int)(e - i * k);
  }
  const int64_t stride = c * 2 * kp;
  float a = 0.0f;
  for (int sp = 0; sp < splits; ++sp) {
    const float* row = partial + sp * stride + i * 2 * kp;
    a += row[j] + row[kp + j];
  }
  G[e] = beta * a;
}

// R (k x k upper, fp64, leading dimension 64): the Cholesky factor of G = L2^T L2
// (G = R^T R) with the decomposition's CholQR rule for dependent columns: a pivot
// d_j = G_jj - sum_{i<j} R_ij^2 not above 1e-12 * max_i G_ii drops column j (row j of R
// zero).  And Rinv (same layout): the inverse of R on the kept rows and columns, zero
// elsewhere, so that L2 Rinv has orthonormal kept columns and zero dropped ones.
// One CTA of 256 threads, everything in shared memory, one barrier per pivot:
//   factorization, j ascending: every thread reads d_j from the diagonal, then every
//     (i, t), j < i <= t, takes A_it -= A_ji A_jt / d_j at once (a thread per entry,
//     through a table of the trailing triangle's entries); rows are scaled at the end;
//   inverse, j descending (R X = I, X starting as the identity): every (i, t),
//     i < j <= t, takes X_it -= R_ij X_jt / R_jj, with row j of X still unscaled; the
//     rows of X are scaled by 1 / R_jj at the end.
constexpr double kLoraDropTol = 1e-12;
constexpr int kLoraCholThreads = 256;
constexpr size_t kLoraCholSmem = (size_t)2 * 64 * 65 * sizeof(double);
__global__ void __launch_bounds__(kLoraCholThreads) lora_chol_kernel(const double* __restrict__ G, int k,
                                                                     double* __restrict__ Rout,
                                                                     double* __restrict__ Rinv) {
  extern __shared__ double lora_smem[];
  double(*A)[65] = reinterpret_cast<double(*)[65]>(lora_smem);
  double(*X)[65] = reinterpret_cast<double(*)[65]>(lora_smem + 64 * 65);
  __shared__ uint16_t pairs[64 * 65 / 2];   // (i << 8) | t over i <= t, rows in descending order
  __shared__ double dinv[64];               // 1 / d_j, 0 for a dropped pivot
  __shared__ double rinv[64];               // 1 / R_jj, 0 for a dropped pivot
  __shared__ double gmax_s;
  const int tid = threadIdx.x;
  for (int e = tid; e < k * k; e += kLoraCholThreads) {
    const int i = e / k, t = e - (e / k) * k;
    A[i][t] = G[e];
    X[i][t] = i == t ? 1.0 : 0.0;
    // rows i' > i come first in the table: they hold (k - 1 - i)(k - i) / 2 entries
    if (i <= t) pairs[(k - 1 - i) * (k - i) / 2 + (t - i)] = (uint16_t)((i << 8) | t);
  }
  if (tid < 32) {
    double g = 0.0;
    for (int j = tid; j < k; j += 32) g = fmax(g, G[j * k + j]);
#pragma unroll
    for (int off = 16; off; off >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, off));
    if (tid == 0) gmax_s = g;
  }
  __syncthreads();
  const double tol = kLoraDropTol * gmax_s;
  for (int j = 0; j < k; ++j) {
    const double d = A[j][j];
    const double di = (!(d > tol) || gmax_s == 0.0) ? 0.0 : 1.0 / d;
    if (tid == 0) dinv[j] = di;
    // the trailing triangle i > j: the first (k - 1 - j)(k - j) / 2 table entries (at most
    // 8 per thread); all loads are issued before any store, so they overlap
    const int cnt = (k - 1 - j) * (k - j) / 2;
    double v[8];
    int at[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = tid + u * kLoraCholThreads;
      at[u] = -1;
      if (e < cnt) {
        const int i = pairs[e] >> 8, t = pairs[e] & 0xFF;
        at[u] = i * 65 + t;
        v[u] = fma(-A[j][i] * di, A[j][t], A[i][t]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (at[u] >= 0) (&A[0][0])[at[u]] = v[u];
    __syncthreads();
  }
  // R_jj = sqrt(d_j), R_jt = A_jt / sqrt(d_j); a dropped row is zero
  for (int e = tid; e < k * k; e += kLoraCholThreads) {
    const int j = e / k, t = e - (e / k) * k;
    if (t >= j) A[j][t] = dinv[j] == 0.0 ? 0.0 : A[j][t] * sqrt(dinv[j]);
  }
  for (int j = tid; j < k; j += kLoraCholThreads) rinv[j] = sqrt(dinv[j]);
  __syncthreads();
  for (int j = k - 1; j > 0; --j) {
    const double ri = rinv[j];
    const int w = k - j;   // j * w <= 1024 entries: at most 4 per thread
    double v[4];
    int at[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = tid + u * kLoraCholThreads;
      at[u] = -1;
      if (e < j * w) {
        const int i = e / w, t = j + (e - (e / w) * w);
        at[u] = i * 65 + t;
        v[u] = fma(-A[i][j] * ri, X[j][t], X[i][t]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (at[u] >= 0) (&X[0][0])[at[u]] = v[u];
    __syncthreads();
  }
  for (int e = tid; e < k * 64; e += kLoraCholThreads) {
    const int i = e / 64, t = e - (e / 64) * 64;
    Rout[e] = (t < k && t >= i) ? A[i][t] : 0.0;
    Rinv[e] = (t < k && t >= i) ? X[i][t] * rinv[i] : 0.0;
  }
}

// In place, a block per 32 rows of L2 (m x k): L2 <- L2 Rinv (Rinv upper triangular,
// leading dimension 64; zero below the diagonal, so full-length sums are exact), fp32
// sums of the fp32-rounded Rinv.  Thread (row r = tid / 8, g = tid % 8) forms the
// outputs j = g, g + 8, ... of its row with independent accumulators.
__global__ void __launch_bounds__(256) lora_times_rinv_kernel(const double* __restrict__ Rinv, int k,
                                                              float* __restrict__ L2, int64_t m) {
  __shared__ float ri[64][65];
  __shared__ float rows[32][65];
  const int64_t r0 = (int64_t)blockIdx.x * 32;
  for (int e = threadIdx.x; e < k * k; e += blockDim.x) {
    const int i = e / k, j = e - (e / k) * k;
    ri[i][j] = (float)Rinv[i * 64 + j];
  }
  for (int e = threadIdx.x; e < 32 * k; e += blockDim.x) {
    const int r = e / k, j = e - (e / k) * k;
    rows[r][j] = r0 + r < m ? L2[(r0 + r) * k + j] : 0.0f;
  }
  __syncthreads();
  const int r = threadIdx.x >> 3, g = threadIdx.x & 7;
  float acc[8] = {};
  for (int i = 0; i < k; ++i) {
    const float x = rows[r][i];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (g + 8 * u < k) acc[u] = fmaf(x, ri[i][g + 8 * u], acc[u]);
  }
  if (r0 + r < m) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (g + 8 * u < k) L2[(r0 + r) * k + g + 8 * u] = acc[u];
  }
}

// In place, a block per 32 columns of L1 (k x n): L1 <- R L1 (R upper triangular, leading
// dimension 64, zero below the diagonal), fp32 sums of the fp32-rounded R.  Lane = column,
// warp w forms the rows j = w, w + 8, ... with independent accumulators.
__global__ void __launch_bounds__(256) lora_left_multiply_kernel(const double* __restrict__ R, int k,
                                                                 float* __restrict__ L1, int64_t n) {
  __shared__ float rs[64][65];
  __shared__ float cols[64][33];
  const int64_t c0 = (int64_t)blockIdx.x * 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < k * k; e += blockDim.x) {
    const int j = e / k, t = e - (e / k) * k;
    rs[j][t] = (float)R[j * 64 + t];
  }
  const bool in = c0 + lane < n;
  for (int t = warp; t < k; t += 8) cols[t][lane] = in ? L1[(int64_t)t * n + c0 + lane] : 0.0f;
  __syncthreads();
  float acc[8] = {};
  for (int t = 0; t < k; ++t) {
    const float x = cols[t][lane];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (warp + 8 * u < k) acc[u] = fmaf(rs[warp + 8 * u][t], x, acc[u]);
  }
  if (in) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (warp + 8 * u < k) L1[(int64_t)(warp + 8 * u) * n + c0 + lane] = acc[u];
  }
}

// W (m x n fp32, leading dimension ldw) += alpha * A B  (A: m x k, B: k x n, fp32, the
// k-term sums in fp32), and Wb = bf16(W) when Wb is given (leading dimension n).  A block
// owns 32 rows x 128 columns; a thread a 4 x 4 tile (rows ty * 4.., columns tx * 4..).
__global__ void __launch_bounds__(256) lowrank_update_kernel(float* __restrict__ W, int64_t ldw, int64_t m,
                                                             int64_t n, const float* __restrict__ A,
                                                             const float* __restrict__ B, int k, float alpha,
                                                             __nv_bfloat16* __restrict__ Wb) {
  __shared__ float a_s[32][65];
  __shared__ __align__(16) float b_s[64][128];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 128;
  for (int e = threadIdx.x; e < 32 * k; e += blockDim.x) {
    const int r = e / k, t = e - (e / k) * k;
    a_s[r][t] = A[(r0 + r) * k + t];
  }
  for (int e = threadIdx.x; e < k * 32; e += blockDim.x) {
    const int t = e / 32, c4 = e - (e / 32) * 32;
    *reinterpret_cast<float4*>(&b_s[t][4 * c4]) = *reinterpret_cast<const float4*>(B + (int64_t)t * n + c0 + 4 * c4);
  }
  __syncthreads();
  const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
  float acc[4][4] = {};
  for (int t = 0; t < k; ++t) {
    const float4 b = *reinterpret_cast<const float4*>(&b_s[t][4 * tx]);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float a = a_s[4 * ty + r][t];
      acc[r][0] = fmaf(a, b.x, acc[r][0]);
      acc[r][1] = fmaf(a, b.y, acc[r][1]);
      acc[r][2] = fmaf(a, b.z, acc[r][2]);
      acc[r][3] = fmaf(a, b.w, acc[r][3]);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = r0 + 4 * ty + r;
    float4* dst = reinterpret_cast<float4*>(W + i * ldw + c0 + 4 * tx);
    float4 w = *dst;
    w.x = fmaf(alpha, acc[r][0], w.x);
    w.y = fmaf(alpha, acc[r][1], w.y);
    w.z = fmaf(alpha, acc[r][2], w.z);
    w.w = fmaf(alpha, acc[r][3], w.w);
    *dst = w;
    if (Wb) {
      uint2 v;
      v.x = pack2(w.x, w.y);
      v.y = pack2(w.z, w.w);
      *reinterpret_cast<uint2*>(Wb + i * n + c0 + 4 * tx) = v;
    }
  }
}

// L1[j][c] = (S[j] / beta) V[c][j]  (k x n from the n x k basis V).
__global__ void lora_set_l1_kernel(const float* __restrict__ S, const float* __restrict__ V, int k, int64_t n,
                                   float beta, float* __restrict__ L1) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)k * n) return;
  const int j = (int)(e / n);
  const int64_t c = e - (int64_t)j * n;
  L1[e] = (S[j] / beta) * V[c * k + j];
}

int lora_pad(int k) { return k <= 32 ? 32 : 64; }

}  // namespace

metis_status run_lora_linear(metis_ctx* ctx, int which, const metis_nvfp4* A, const metis_nvfp4* B,
                             const metis_matrix* M, const float* L2, const float* L1, int k, float beta, float* T,
                             void* C, int64_t ldc, int32_t c_dtype) {
  const int64_t p = A->outer, K = A->inner, q = B->outer;
  const int kp = lora_pad(k);
  const int fold_k = 2 * kp;   // 64 or 128
  // forward: Lin = L2 (K x k), Lout(c, j) = L1[j][c]; input gradient: Lin = L1^T (L1 is k x K),
  // Lout(c, j) = L2[c][j]
  const float* Lin = which == 0 ? L2 : L1;
  const float* Lout = which == 0 ? L1 : L2;
  const int splits = normalize_splits(K, bf16_splits(ctx, p, K, kp));
  const size_t need = (size_t)kp * K * 2 + (size_t)splits * p * kp * 4 + (size_t)p * fold_k * 2 +
                      (size_t)q * fold_k * 2 + 4 * 256;
  metis_status s = ensure_workspace(ctx, need);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  auto* Bt = static_cast<__nv_bfloat16*>(ws.take((size_t)kp * K * 2));
  auto* Tp = static_cast<float*>(ws.take((size_t)splits * p * kp * 4));
  auto* Fa = static_cast<__nv_bfloat16*>(ws.take((size_t)p * fold_k * 2));
  auto* Fb = static_cast<__nv_bfloat16*>(ws.take((size_t)q * fold_k * 2));
  if (!Fb) return fail(ctx, METIS_ERR_WORKSPACE, "LoRA workspace layout");
  cudaStream_t st = ctx->stream;
  lora_pack_in_kernel<<<blocks_of((int64_t)kp * K), 256, 0, st>>>(Lin, which != 0, K, k, kp, Bt);
  count_launch();
  if ((s = check_cuda(ctx, cudaGetLastError(), "LoRA factor packing")) != METIS_OK) return s;
  // T = M Lin on the bf16 tensor cores (split-K fp32 partials)
  if ((s = launch_gemm_bf16(ctx, M->data, M->ld, p, Bt, K, kp, K, Tp, kp, splits)) != METIS_OK) return s;
  lora_fold_kernel<<<(unsigned)(p / kLoraRows + q / kLoraRows), 256, 0, st>>>(
      Tp, splits, p, k, kp, beta, A->tensor_scale, B->tensor_scale, Lout, which == 0, q, fold_k, T, Fa, Fb);
  count_launch();
  if ((s = check_cuda(ctx, cudaGetLastError(), "LoRA fold operands")) != METIS_OK) return s;
  GemmArgs g{A, B, Fa, Fb, fold_k, nullptr, C, ldc, c_dtype, 1.0f, q, 1, 0};
  return launch_gemm_nvfp4(ctx, g);
}

metis_status run_lora_branch_grad(metis_ctx* ctx, const metis_matrix* M, const float* T, int k, float beta,
                                  bool transpose_out, float* G) {
  const int64_t p = M->rows, c = M->cols;
  const int kp = lora_pad(k);
  const int splits = normalize_splits(p, bf16_splits(ctx, c, p, 2 * kp));
  const size_t need = (size_t)c * p * 2 + (size_t)2 * kp * p * 2 + (size_t)splits * c * 2 * kp * 4 + 4 * 256;
  metis_status s = ensure_workspace(ctx, need);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  void* Mt = ws.take((size_t)c * p * 2);
  void* Tt = ws.take((size_t)2 * kp * p * 2);
  auto* part = static_cast<float*>(ws.take((size_t)splits * c * 2 * kp * 4));
  if (!part) return fail(ctx, METIS_ERR_WORKSPACE, "LoRA gradient workspace layout");
  cudaStream_t st = ctx->stream;
  cudaError_t e = launch_transpose_bf16(M->data, M->ld, p, c, Mt, st);
  if (e == cudaSuccess) e = launch_split_hi_lo_t(T, p, k, kp, Tt, st);
  if ((s = check_cuda(ctx, e, "LoRA gradient operands")) != METIS_OK) return s;
  // M^T T with T as a bf16 hi/lo pair: (c x p) x (p x 2 kp)
  if ((s = launch_gemm_bf16(ctx, Mt, p, c, Tt, p, 2 * kp, p, part, 2 * kp, splits)) != METIS_OK) return s;
  lora_grad_reduce_kernel<<<blocks_of(c * k), 256, 0, st>>>(part, splits, c, kp, k, beta, transpose_out, G);
  count_launch();
  return check_cuda(ctx, cudaGetLastError(), "LoRA gradient reduction");
}

metis_status run_lora_constrain(metis_ctx* ctx, float* L2, int64_t m, float* L1, int64_t n, int k) {
  const size_t nd = gram_scratch_doubles(ctx, k);
  metis_status s = ensure_workspace(ctx, nd * 8 + (size_t)2 * 64 * 64 * 8 + 3 * 256);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  auto* scratch = static_cast<double*>(ws.take(nd * 8));
  auto* R = static_cast<double*>(ws.take((size_t)64 * 64 * 8));
  auto* Rinv = static_cast<double*>(ws.take((size_t)64 * 64 * 8));
  if (!Rinv) return fail(ctx, METIS_ERR_WORKSPACE, "LoRA constraint workspace layout");
  cudaStream_t st = ctx->stream;
  double* G = nullptr;
  if ((s = launch_gram(ctx, L2, m, k, scratch, &G)) != METIS_OK) return s;
  cudaError_t e = cudaFuncSetAttribute(lora_chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kLoraCholSmem);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(lora_chol_kernel)");
  lora_chol_kernel<<<1, kLoraCholThreads, kLoraCholSmem, st>>>(G, k, R, Rinv);
  lora_times_rinv_kernel<<<blocks_of(m, 32), 256, 0, st>>>(Rinv, k, L2, m);
  lora_left_multiply_kernel<<<blocks_of(n, 32), 256, 0, st>>>(R, k, L1, n);
  count_launch(3);
  return check_cuda(ctx, cudaGetLastError(), "LoRA constraint");
}

metis_status run_lora_realign(metis_ctx* ctx, float* W, int64_t m, int64_t n, int64_t ldw, float* L2, float* L1,
                              int k, float beta, const metis_decomp_params* p, uint32_t step, metis_factors* f,
                              void* W_bf16) {
  cudaStream_t st = ctx->stream;
  const dim3 grid((unsigned)(n / 128), (unsigned)(m / 32));
  // W_eff = W_res + beta L2 L1, and its bf16 copy for the decomposition
  lowrank_update_kernel<<<grid, 256, 0, st>>>(W, ldw, m, n, L2, L1, k, beta,
                                               static_cast<__nv_bfloat16*>(W_bf16));
  count_launch();
  metis_status s = check_cuda(ctx, cudaGetLastError(), "LoRA realignment (W_eff)");
  if (s != METIS_OK) return s;
  const metis_matrix Mb{W_bf16, m, n, n};
  if ((s = run_decompose(ctx, &Mb, p, 1, step, f)) != METIS_OK) return s;
  cudaError_t e = cudaMemcpyAsync(L2, f->U, (size_t)m * k * 4, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) {
    lora_set_l1_kernel<<<blocks_of((int64_t)k * n), 256, 0, st>>>(f->S, f->V, k, n, beta, L1);
    count_launch();
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    // W_res = W_eff - beta L2 L1
    lowrank_update_kernel<<<grid, 256, 0, st>>>(W, ldw, m, n, L2, L1, k, -beta, nullptr);
    count_launch();
    e = cudaGetLastError();
  }
  return check_cuda(ctx, e, "LoRA realignment");
}

}  // namespace metis
