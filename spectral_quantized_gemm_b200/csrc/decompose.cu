// Randomized spectral decomposition M ~ U S V^T with a reused basis.
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes):
// key design 2 -- estimate the dominant subspace from l_k << l randomly sampled
// rows and a Gaussian test matrix Omega of width k + s (randomized SVD); key
// design 3 -- reuse the low-rank factors across steps, refreshing every few
// steps; training strategy -- rank 1.5%, refresh every 8 steps.
//
// refresh:  rows <- l_k smallest Philox keys;  Omega <- Box-Muller(Philox);
//           Y = M_s Omega;  Q = Y R^+ (CholQR);  Bm^T = M_s^T Q;
//           R2 = chol(Bm Bm^T);  Jacobi SVD of R2^T;  V = Bm^T R2^+ W'[:, :k]
// every step: P = M V;  R = chol(P^T P);  Jacobi SVD R = U_r S_r V_r^T;
//           U = P R^+ U_r;  S = S_r;  V <- V V_r;  sign fix;  NVFP4 of U^T, V^T
// The small dense steps (Cholesky with dependent-column drop, triangular
// pseudo-inverse, one-sided Jacobi SVD, sorting) run in one CTA in fp64.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"

namespace metis {
namespace {

constexpr double kDropTol = 1e-12;
constexpr double kJacobiTol = 1e-12;
constexpr int kJacobiMaxSweeps = 40;
constexpr int kMaxW = 128;
constexpr size_t kSmallSmemMax = 200 * 1024;  // dynamic shared memory of the small solver

// ---------------------------------------------------------------- sampling
__global__ void sample_keys_kernel(int64_t rows, uint64_t seed, uint32_t tag, uint32_t step, uint64_t* keys) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  const Words4 w = stream_call(seed, tag, step, (uint64_t)i >> 2);
  keys[i] = ((uint64_t)w.w[i & 3] << 32) | (uint64_t)i;
}

// One CTA: radix-select the l_k smallest keys, emit their row indices ascending.
__global__ void __launch_bounds__(1024) sample_select_kernel(const uint64_t* keys, int64_t rows, int l_k,
                                                             int32_t* out_idx) {
  __shared__ unsigned int hist[256];
  __shared__ uint64_t prefix, mask;
  __shared__ int64_t need;
  __shared__ int64_t scan[1024];
  if (threadIdx.x == 0) {
    prefix = 0;
    mask = 0;
    need = l_k;
  }
  __syncthreads();
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint64_t pf = prefix, mk = mask;
    for (int64_t i = threadIdx.x; i < rows; i += blockDim.x) {
      const uint64_t key = keys[i];
      if ((key & mk) == pf) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int64_t cum = 0;
      int b = 0;
      for (; b < 256; ++b) {
        if (cum + hist[b] >= need) break;
        cum += hist[b];
      }
      need -= cum;
      prefix |= (uint64_t)b << shift;
      mask |= (uint64_t)255u << shift;
    }
    __syncthreads();
  }
  const uint64_t thr = prefix;  // the l_k-th smallest key; keys are distinct
  const int64_t chunk = (rows + blockDim.x - 1) / blockDim.x;
  const int64_t lo = threadIdx.x * chunk, hi = min(rows, lo + chunk);
  int64_t cnt = 0;
  for (int64_t i = lo; i < hi; ++i) cnt += keys[i] <= thr;
  scan[threadIdx.x] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t acc = 0;
    for (int t = 0; t < (int)blockDim.x; ++t) {
      const int64_t c = scan[t];
      scan[t] = acc;
      acc += c;
    }
  }
  __syncthreads();
  int64_t pos = scan[threadIdx.x];
  for (int64_t i = lo; i < hi; ++i)
    if (keys[i] <= thr) out_idx[pos++] = (int32_t)i;
}

__global__ void iota_kernel(int64_t n, int32_t* out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = (int32_t)i;
}

// ---------------------------------------------------------------- Omega
__global__ void omega_kernel(int64_t n, uint64_t seed, uint32_t tag, uint32_t step, float* out, float* copy) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t * 4 >= n) return;
  const Words4 w = stream_call(seed, tag, step, (uint64_t)t);
  double z[4];
#pragma unroll
  for (int pair = 0; pair < 2; ++pair) {
    const double u1 = ((double)w.w[2 * pair] + 1.0) * 0x1p-32;
    const double u2 = (double)w.w[2 * pair + 1] * 0x1p-32;
    const double rad = sqrt(-2.0 * log(u1));
    const double ang = 6.283185307179586476925286766559 * u2;
    z[2 * pair] = rad * cos(ang);
    z[2 * pair + 1] = rad * sin(ang);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t e = t * 4 + i;
    if (e < n) {
      const float v = (float)z[i];
      out[e] = v;
      if (copy) copy[e] = v;
    }
  }
}

// ------------------------------------------------ skinny products (fp32 accumulate)
// Partial C[r][j] = sum_{c in chunk} M[rowmap[r]][c] * B[c][j]   (M bf16, B fp32 n x w)
// grid: (ceil(nr/64), nsplit), block 256; partial layout [split][nr][w]
constexpr int kRowsPerBlock = 64;
constexpr int kColChunk = 32;
__global__ void rows_times_matrix_kernel(const __nv_bfloat16* __restrict__ M, int64_t ld, const int32_t* rowmap,
                                         int64_t nr, int64_t ncols, const float* __restrict__ B, int w,
                                         int64_t split_len, float* __restrict__ partial, uint32_t* status) {
  __shared__ float sm[kRowsPerBlock][kColChunk + 1];
  __shared__ float sb[kColChunk][kMaxW];
  const int64_t r0 = (int64_t)blockIdx.x * kRowsPerBlock;
  const int64_t c_begin = (int64_t)blockIdx.y * split_len;
  const int64_t c_end = min(ncols, c_begin + split_len);
  const int nout = kRowsPerBlock * w;
  float acc[(kRowsPerBlock * kMaxW) / 256];
  const int per = (nout + 255) / 256;
  for (int i = 0; i < per; ++i) acc[i] = 0.0f;
  bool finite = true;
  for (int64_t c0 = c_begin; c0 < c_end; c0 += kColChunk) {
    for (int e = threadIdx.x; e < kRowsPerBlock * kColChunk; e += blockDim.x) {
      const int r = e / kColChunk, c = e % kColChunk;
      const int64_t row = r0 + r;
      float v = 0.0f;
      if (row < nr && c0 + c < c_end) {
        const int64_t src = rowmap ? rowmap[row] : row;
        v = __bfloat162float(M[src * ld + c0 + c]);
        finite &= isfinite(v);
      }
      sm[r][c] = v;
    }
    for (int e = threadIdx.x; e < kColChunk * w; e += blockDim.x) {
      const int c = e / w, j = e % w;
      sb[c][j] = (c0 + c < c_end) ? B[(c0 + c) * w + j] : 0.0f;
    }
    __syncthreads();
    for (int i = 0; i < per; ++i) {
      const int o = threadIdx.x + i * 256;
      if (o < nout) {
        const int r = o / w, j = o % w;
        float a = acc[i];
#pragma unroll 8
        for (int c = 0; c < kColChunk; ++c) a = fmaf(sm[r][c], sb[c][j], a);
        acc[i] = a;
      }
    }
    __syncthreads();
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  for (int i = 0; i < per; ++i) {
    const int o = threadIdx.x + i * 256;
    if (o < nout) {
      const int r = o / w, j = o % w;
      if (r0 + r < nr) partial[((int64_t)blockIdx.y * nr + r0 + r) * w + j] = acc[i];
    }
  }
}

// out[e] = sum over splits in order (deterministic).
__global__ void sum_splits_kernel(const float* partial, int nsplit, int64_t n, float* out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float a = 0.0f;
  for (int s = 0; s < nsplit; ++s) a += partial[(int64_t)s * n + e];
  out[e] = a;
}

// Bm^T = M_s^T Q: out[c][j] = sum_r M[rowmap[r]][c] * Q[r][j]   (64 columns of M per block)
__global__ void cols_times_matrix_kernel(const __nv_bfloat16* __restrict__ M, int64_t ld, const int32_t* rowmap,
                                         int64_t nr, int64_t ncols, const float* __restrict__ Q, int w,
                                         float* __restrict__ out) {
  __shared__ float sm[16][65];
  __shared__ float sq[16][kMaxW];
  const int64_t c0 = (int64_t)blockIdx.x * 64;
  const int nout = 64 * w;
  const int per = (nout + 255) / 256;
  float acc[(64 * kMaxW) / 256];
  for (int i = 0; i < per; ++i) acc[i] = 0.0f;
  for (int64_t r0 = 0; r0 < nr; r0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += blockDim.x) {
      const int r = e / 64, c = e % 64;
      float v = 0.0f;
      if (r0 + r < nr && c0 + c < ncols) {
        const int64_t src = rowmap ? rowmap[r0 + r] : r0 + r;
        v = __bfloat162float(M[src * ld + c0 + c]);
      }
      sm[r][c] = v;
    }
    for (int e = threadIdx.x; e < 16 * w; e += blockDim.x) {
      const int r = e / w, j = e % w;
      sq[r][j] = (r0 + r < nr) ? Q[(r0 + r) * w + j] : 0.0f;
    }
    __syncthreads();
    for (int i = 0; i < per; ++i) {
      const int o = threadIdx.x + i * 256;
      if (o < nout) {
        const int c = o / w, j = o % w;
        float a = acc[i];
#pragma unroll
        for (int r = 0; r < 16; ++r) a = fmaf(sm[r][c], sq[r][j], a);
        acc[i] = a;
      }
    }
    __syncthreads();
  }
  for (int i = 0; i < per; ++i) {
    const int o = threadIdx.x + i * 256;
    if (o < nout) {
      const int c = o / w, j = o % w;
      if (c0 + c < ncols) out[(c0 + c) * w + j] = acc[i];
    }
  }
}

// C (n x k2, fp32) = A (n x k1, fp32 row-major) * T (k1 x k2, fp64 row-major, ld kMaxW)
__global__ void times_small_kernel(const float* __restrict__ A, int64_t n, int k1, const double* __restrict__ T,
                                   int k2, float* __restrict__ C) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n * k2) return;
  const int64_t i = e / k2;
  const int j = (int)(e - i * k2);
  double a = 0.0;
  for (int t = 0; t < k1; ++t) a = fma((double)A[i * k1 + t], T[t * kMaxW + j], a);
  C[e] = (float)a;
}

// --------------------------------------------------------------- Gram (fp64)
// partial[block] = A_rows^T A_rows over the block's rows (chunks of 32 staged in
// shared memory); upper triangle, full w x w storage.  Each thread keeps its
// (a, b) sums in registers across the chunks.
constexpr int kGramRows = 32;
constexpr int kGramPer = 64;   // (w*w)/256 for w <= 128
__global__ void gram_partial_kernel(const float* __restrict__ A, int64_t n, int w, int64_t rows_per_block,
                                    double* partial, uint32_t* status) {
  __shared__ double sa[kGramRows][kMaxW + 1];
  const int64_t r_begin = (int64_t)blockIdx.x * rows_per_block;
  const int64_t r_end = min(n, r_begin + rows_per_block);
  double acc[kGramPer];
#pragma unroll
  for (int i = 0; i < kGramPer; ++i) acc[i] = 0.0;
  bool finite = true;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kGramRows) {
    __syncthreads();
    for (int e = threadIdx.x; e < kGramRows * w; e += blockDim.x) {
      const int r = e / w, j = e % w;
      const float v = (r0 + r < r_end) ? A[(r0 + r) * w + j] : 0.0f;
      finite &= isfinite(v);
      sa[r][j] = v;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kGramPer; ++i) {
      const int e = threadIdx.x + i * 256;
      if (e < w * w) {
        const int a = e / w, b = e % w;
        if (a <= b) {
          double s2 = acc[i];
#pragma unroll 8
          for (int r = 0; r < kGramRows; ++r) s2 = fma(sa[r][a], sa[r][b], s2);
          acc[i] = s2;
        }
      }
    }
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
#pragma unroll
  for (int i = 0; i < kGramPer; ++i) {
    const int e = threadIdx.x + i * 256;
    if (e < w * w) partial[(int64_t)blockIdx.x * w * w + e] = acc[i];
  }
}

__global__ void gram_reduce_kernel(const double* partial, int nblocks, int w, double* G) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= w * w) return;
  const int a = e / w, b = e % w;
  double acc = 0.0;
  const int src = a <= b ? e : b * w + a;
  for (int c = 0; c < nblocks; ++c) acc += partial[(int64_t)c * w * w + src];
  G[e] = acc;
}

// ----------------------------------------------------- single-CTA small solver
// Modes: 0 = CholQR factor only (T = R^+), 1 = refresh SVD (T = R^+ W'[:, :k] with
// SVD of R^T), 2 = step SVD (T = R^+ U_r[:, :k], Vr, S from SVD of R).
// Shared memory holds the n x n matrix being orthogonalized, stored by columns;
// R^+ and the accumulated rotations live in (L2-resident) workspace.
struct SmallOut {
  double* T;      // n x kMaxW (row-major, ld kMaxW)
  double* Vr;     // n x kMaxW
  float* S;       // k
  int* flags;     // [0] = numeric failure
  double* Rinv;   // kMaxW x kMaxW scratch
  double* Vt;     // kMaxW x kMaxW scratch: accumulated rotations, by columns
};

__global__ void __launch_bounds__(1024) small_solver_kernel(const double* __restrict__ G, int n, int k, int mode,
                                                            SmallOut out, uint32_t* status) {
  extern __shared__ double At[];      // ld x ld; Cholesky factor first, then A by columns
  __shared__ int dropped[kMaxW];
  __shared__ double gmax_s, pivot_s;
  __shared__ double sig[kMaxW];
  __shared__ int order[kMaxW];
  __shared__ int any_rot;
  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int ne = (n + 1) & ~1;
  const int ld = ne;
  double* R = At;                     // R[i * ld + j], upper triangular
  double* Rinv = out.Rinv;            // ld kMaxW
  // accumulated rotations by columns: in shared memory after the matrix when
  // both fit, else in the (L2-resident) workspace
  const bool vt_shared = (size_t)2 * ld * ld * sizeof(double) <= kSmallSmemMax;
  double* Vt = vt_shared ? At + ld * ld : out.Vt;
  const int vld = vt_shared ? ld : kMaxW;
  __shared__ double nrm[kMaxW];

  for (int e = tid; e < ld * ld; e += nt) R[e] = 0.0;
  for (int e = tid; e < kMaxW * kMaxW; e += nt) Rinv[e] = 0.0;
  if (tid == 0) {
    double g = 0.0;
    for (int j = 0; j < n; ++j) g = fmax(g, G[j * n + j]);
    gmax_s = g;
  }
  __syncthreads();
  const double tol = kDropTol * gmax_s;
  // Cholesky G = R^T R with dependent columns dropped (their row of R is zero)
  for (int j = 0; j < n; ++j) {
    if (tid == 0) {
      double d = G[j * n + j];
      for (int i = 0; i < j; ++i) d -= R[i * ld + j] * R[i * ld + j];
      const bool drop = !(d > tol) || gmax_s == 0.0;
      dropped[j] = drop;
      pivot_s = drop ? 0.0 : sqrt(d);
      R[j * ld + j] = pivot_s;
    }
    __syncthreads();
    if (!dropped[j]) {
      for (int t = j + 1 + tid; t < n; t += nt) {
        double v = G[j * n + t];
        for (int i = 0; i < j; ++i) v -= R[i * ld + j] * R[i * ld + t];
        R[j * ld + t] = v / pivot_s;
      }
    }
    __syncthreads();
  }
  // R^+: column j solves R x = e_j on the kept indices
  for (int j = tid; j < n; j += nt) {
    if (dropped[j]) continue;
    Rinv[j * kMaxW + j] = 1.0 / R[j * ld + j];
    for (int i = j - 1; i >= 0; --i) {
      if (dropped[i]) continue;
      double acc = 0.0;
      for (int t = i + 1; t <= j; ++t) acc += R[i * ld + t] * Rinv[t * kMaxW + j];
      Rinv[i * kMaxW + j] = -acc / R[i * ld + i];
    }
  }
  __syncthreads();
  if (mode == 0) {
    for (int e = tid; e < n * n; e += nt) out.T[(e / n) * kMaxW + e % n] = Rinv[(e / n) * kMaxW + e % n];
    return;
  }
  // A by columns: mode 1 takes A = R^T, whose column j is row j of R (already the
  // layout); mode 2 takes A = R, so transpose in place.
  if (mode == 2) {
    for (int e = tid; e < ld * ld; e += nt) {
      const int i = e / ld, j = e % ld;
      if (i < j) {
        const double a = R[i * ld + j];
        R[i * ld + j] = R[j * ld + i];
        R[j * ld + i] = a;
      }
    }
  }
  for (int e = tid; e < vld * vld; e += nt) Vt[e] = ((e / vld) == (e % vld) && (e / vld) < ne) ? 1.0 : 0.0;
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const int npairs = ne / 2;
  int sweep = 0;
  for (; sweep < kJacobiMaxSweeps; ++sweep) {
    if (tid == 0) any_rot = 0;
    // exact column norms at the start of every sweep; within the sweep they are
    // updated with each rotation (||a_p||^2 -= t g, ||a_q||^2 += t g)
    for (int j = tid; j < ne; j += nt) {
      double s2 = 0.0;
      for (int r = 0; r < ne; ++r) s2 = fma(At[j * ld + r], At[j * ld + r], s2);
      nrm[j] = s2;
    }
    __syncthreads();
    for (int round = 0; round < ne - 1; ++round) {
      for (int pr = warp; pr < npairs; pr += nwarps) {
        // round-robin tournament: position 0 stays, the others rotate each round
        const int pa = pr, pb = ne - 1 - pr;
        int p = pa == 0 ? 0 : 1 + (pa - 1 + round) % (ne - 1);
        int q = pb == 0 ? 0 : 1 + (pb - 1 + round) % (ne - 1);
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        double* cp = At + p * ld;
        double* cq = At + q * ld;
        const double al = nrm[p], be = nrm[q];
        double ga = 0.0;
        for (int r = lane; r < ne; r += 32) ga = fma(cp[r], cq[r], ga);
#pragma unroll
        for (int off = 16; off; off >>= 1) ga += __shfl_xor_sync(0xffffffffu, ga, off);
        if (ga != 0.0 && fabs(ga) > kJacobiTol * sqrt(al * be)) {
          const double zeta = (be - al) / (2.0 * ga);
          const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          const double c = 1.0 / sqrt(1.0 + t * t), s = c * t;
          double* vp = Vt + p * vld;
          double* vq = Vt + q * vld;
          for (int r = lane; r < ne; r += 32) {
            const double x = cp[r], y = cq[r];
            cp[r] = c * x - s * y;
            cq[r] = s * x + c * y;
            const double vx = vp[r], vy = vq[r];
            vp[r] = c * vx - s * vy;
            vq[r] = s * vx + c * vy;
          }
          if (lane == 0) {
            any_rot = 1;
            nrm[p] = al - t * ga;
            nrm[q] = be + t * ga;
          }
        }
      }
      __syncthreads();
    }
    if (!any_rot) break;
    __syncthreads();
  }
  if (sweep == kJacobiMaxSweeps && tid == 0) {
    raise_status(status, METIS_DEV_NUMERIC);
    out.flags[0] = 1;
  }
  // singular values and descending order (ties by index)
  for (int j = tid; j < ne; j += nt) {
    double s2 = 0.0;
    for (int r = 0; r < ne; ++r) s2 = fma(At[j * ld + r], At[j * ld + r], s2);
    sig[j] = sqrt(s2);
  }
  __syncthreads();
  for (int j = tid; j < ne; j += nt) {
    int rank = 0;
    for (int i = 0; i < ne; ++i) rank += (sig[i] > sig[j]) || (sig[i] == sig[j] && i < j);
    order[rank] = j;
  }
  __syncthreads();
  if (mode == 1) {
    // T = R^+ W'[:, top k]  (n x k), W' the accumulated rotations
    for (int e = tid; e < n * k; e += nt) {
      const int i = e / k, c = e % k;
      const double* wcol = Vt + order[c] * vld;
      double a = 0.0;
      for (int t = 0; t < n; ++t) a = fma(Rinv[i * kMaxW + t], wcol[t], a);
      out.T[i * kMaxW + c] = a;
    }
  } else {
    // U_r = A / sigma (zero column for sigma == 0); T = R^+ U_r[:, top k]; Vr; S
    for (int e = tid; e < n * k; e += nt) {
      const int i = e / k, c = e % k;
      const int src = order[c];
      const double sg = sig[src];
      double a = 0.0;
      if (sg > 0.0)
        for (int t = 0; t < n; ++t) a = fma(Rinv[i * kMaxW + t], At[src * ld + t] / sg, a);
      out.T[i * kMaxW + c] = a;
      out.Vr[i * kMaxW + c] = Vt[src * vld + i];
    }
    for (int c = tid; c < k; c += nt) out.S[c] = (float)sig[order[c]];
  }
}

// ------------------------------------------- tensor-core projection helpers
// out (2kp x n, bf16 row-major): row j < k = hi(F[:, j]), row kp + j = lo(F[:, j]) with
// hi = bf16(F), lo = bf16(F - hi); other rows zero.  F is n x k fp32 row-major.
__global__ void split_hi_lo_t_kernel(const float* __restrict__ F, int64_t n, int k, int kp,
                                     __nv_bfloat16* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)2 * kp * n) return;
  const int j = (int)(e / n);
  const int64_t i = e - (int64_t)j * n;
  const int jj = j < kp ? j : j - kp;
  float v = 0.0f;
  if (jj < k) {
    const float f = F[i * k + jj];
    const __nv_bfloat16 hi = __float2bfloat16_rn(f);
    v = j < kp ? __bfloat162float(hi) : f - __bfloat162float(hi);
  }
  out[e] = __float2bfloat16_rn(v);
}

// out[i][j] = sum over splits (in order) of partial[s][i][j] + partial[s][i][kp + j],  j < k.
__global__ void reduce_hi_lo_kernel(const float* __restrict__ partial, int splits, int64_t rows, int kp, int k,
                                    float* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= rows * k) return;
  const int64_t i = e / k;
  const int j = (int)(e - i * k);
  const int64_t stride = rows * 2 * kp;
  float a = 0.0f;
  for (int sp = 0; sp < splits; ++sp) {
    const float* row = partial + sp * stride + i * 2 * kp;
    a += row[j] + row[kp + j];
  }
  out[e] = a;
}

int pad_width(int w) { return w <= 16 ? 16 : w <= 32 ? 32 : w <= 64 ? 64 : 128; }

// ------------------------------------------------------------- sign fix
// flip[j] = 1 if the largest-|.| entry of column j of V (first index on ties) is negative.
__global__ void sign_pick_kernel(const float* __restrict__ V, int64_t n, int k, int* flip) {
  const int j = blockIdx.x;
  float best = -1.0f;
  int64_t bi = 0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const float a = fabsf(V[i * k + j]);
    if (a > best) {
      best = a;
      bi = i;
    }
  }
  __shared__ float sb[256];
  __shared__ int64_t si[256];
  sb[threadIdx.x] = best;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int s = blockDim.x / 2; s; s >>= 1) {
    if (threadIdx.x < s) {
      const float ob = sb[threadIdx.x + s];
      const int64_t oi = si[threadIdx.x + s];
      if (ob > sb[threadIdx.x] || (ob == sb[threadIdx.x] && oi < si[threadIdx.x])) {
        sb[threadIdx.x] = ob;
        si[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) flip[j] = V[si[0] * k + j] < 0.0f;
}

__global__ void apply_flip_kernel(const float* __restrict__ src, int64_t n, int k, const int* flip, float* dst) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n * k) return;
  const int j = (int)(e % k);
  dst[e] = flip[j] ? -src[e] : src[e];
}

unsigned blocks_for(int64_t n, int t = 256) { return (unsigned)((n + t - 1) / t); }

}  // namespace

metis_status run_decompose(metis_ctx* ctx, const metis_matrix* M, const metis_decomp_params* p, int refresh,
                           uint32_t step, metis_factors* f) {
  const int64_t r = M->rows, c = M->cols;
  const int k = p->k, w = p->k + p->s;
  const int64_t lk = p->l_k;
  const __nv_bfloat16* Mb = static_cast<const __nv_bfloat16*>(M->data);
  cudaStream_t st = ctx->stream;

  // split the long dimension of the skinny products into chunks of ~1024 columns
  const int64_t split_len = 1024;
  const int nsplit = (int)((c + split_len - 1) / split_len);
  const int64_t rows_needed = std::max(r, lk);
  size_t need = 0;
  need += (size_t)r * 8 + 256;                                    // keys
  need += (size_t)lk * 4 + 256;                                   // idx
  need += (size_t)c * w * 4 + 256;                                // Omega
  need += (size_t)nsplit * rows_needed * std::max(w, k) * 4 + 256;  // partials
  need += (size_t)rows_needed * std::max(w, k) * 4 + 256;         // Y / P
  need += (size_t)rows_needed * std::max(w, k) * 4 + 256;         // Q / U
  need += (size_t)c * std::max(w, k) * 4 + 256;                   // Bm^T / V new
  need += (size_t)((std::max(rows_needed, c) + kGramRows - 1) / kGramRows) * w * w * 8 + 256;  // gram partials
  need += (size_t)kMaxW * kMaxW * 8 * 5 + 2048;                   // G, T, Vr, Rinv, Vt
  need += 64 * 4 * 3 + 1024;                                      // S, flags, flips
  const int kpw = pad_width(std::max(w, k));
  need += (size_t)2 * kpw * c * 2 + 256;                          // hi/lo transposed operand
  const int splits_est = normalize_splits(c, bf16_splits(ctx, r, c));
  const size_t tc_partial_bytes = (size_t)splits_est * r * 2 * kpw * 4;
  need += tc_partial_bytes + 256;                                 // split partials
  metis_status s = ensure_workspace(ctx, need);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  uint64_t* keys = static_cast<uint64_t*>(ws.take((size_t)r * 8));
  int32_t* idx = static_cast<int32_t*>(ws.take((size_t)lk * 4));
  float* omega = static_cast<float*>(ws.take((size_t)c * w * 4));
  float* partial = static_cast<float*>(ws.take((size_t)nsplit * rows_needed * std::max(w, k) * 4));
  float* Y = static_cast<float*>(ws.take((size_t)rows_needed * std::max(w, k) * 4));
  float* Q = static_cast<float*>(ws.take((size_t)rows_needed * std::max(w, k) * 4));
  float* Bt = static_cast<float*>(ws.take((size_t)c * std::max(w, k) * 4));
  double* gpart = static_cast<double*>(
      ws.take((size_t)((std::max(rows_needed, c) + kGramRows - 1) / kGramRows) * w * w * 8));
  double* G = static_cast<double*>(ws.take((size_t)kMaxW * kMaxW * 8));
  double* T = static_cast<double*>(ws.take((size_t)kMaxW * kMaxW * 8));
  double* Vr = static_cast<double*>(ws.take((size_t)kMaxW * kMaxW * 8));
  double* Rinv = static_cast<double*>(ws.take((size_t)kMaxW * kMaxW * 8));
  double* Vt = static_cast<double*>(ws.take((size_t)kMaxW * kMaxW * 8));
  float* Sw = static_cast<float*>(ws.take(64 * 4));
  int* flags = static_cast<int*>(ws.take(64 * 4));
  int* flip = static_cast<int*>(ws.take(64 * 4));
  __nv_bfloat16* bt2 = static_cast<__nv_bfloat16*>(ws.take((size_t)2 * kpw * c * 2));
  float* tc_partial = static_cast<float*>(ws.take(tc_partial_bytes));
  if (!tc_partial) return fail(ctx, METIS_ERR_WORKSPACE, "decompose workspace layout");

  const int ne_max = ((std::max(w, k) + 1) & ~1);
  const size_t small_smem = std::max((size_t)ne_max * ne_max * 8,
                                     std::min(kSmallSmemMax, (size_t)2 * ne_max * ne_max * 8));
  cudaError_t e = cudaFuncSetAttribute(small_solver_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)small_smem);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(small solver)");
  SmallOut so{T, Vr, Sw, flags, Rinv, Vt};

  auto gram = [&](const float* A, int64_t n, int width) {
    const int64_t chunks = (n + kGramRows - 1) / kGramRows;
    const int64_t per_block = ((chunks + ctx->sm_count - 1) / ctx->sm_count) * kGramRows;
    const int nb = (int)((n + per_block - 1) / per_block);
    gram_partial_kernel<<<nb, 256, 0, st>>>(A, n, width, per_block, gpart, ctx->status); count_launch();
    gram_reduce_kernel<<<blocks_for((int64_t)width * width), 256, 0, st>>>(gpart, nb, width, G); count_launch();
  };
  // out (r x width) = M B on the tensor cores: B (c x width fp32) as a bf16 hi/lo pair
  auto project = [&](const float* B, int width, float* out) -> metis_status {
    const int kp = pad_width(width);
    split_hi_lo_t_kernel<<<blocks_for((int64_t)2 * kp * c), 256, 0, st>>>(B, c, width, kp, bt2); count_launch();
    const int splits = normalize_splits(c, bf16_splits(ctx, r, c));
    if ((size_t)splits * r * 2 * kp * 4 > tc_partial_bytes)
      return fail(ctx, METIS_ERR_WORKSPACE, "projection partials exceed workspace");
    metis_status st2 = launch_gemm_bf16(ctx, Mb, M->ld, r, bt2, c, 2 * kp, c, tc_partial, 2 * kp, splits);
    if (st2 != METIS_OK) return st2;
    reduce_hi_lo_kernel<<<blocks_for(r * width), 256, 0, st>>>(tc_partial, splits, r, kp, width, out); count_launch();
    return METIS_OK;
  };
  auto rows_times = [&](const int32_t* rowmap, int64_t nr, const float* B, int width, float* out) {
    dim3 grid(blocks_for(nr, kRowsPerBlock), nsplit);
    rows_times_matrix_kernel<<<grid, 256, 0, st>>>(Mb, M->ld, rowmap, nr, c, B, width, split_len, partial,
                                                   ctx->status); count_launch();
    sum_splits_kernel<<<blocks_for(nr * width), 256, 0, st>>>(partial, nsplit, nr * width, out); count_launch();
  };

  if (refresh) {
    const bool sampled = lk < r;
    if (sampled) {
      sample_keys_kernel<<<blocks_for(r), 256, 0, st>>>(r, p->seed, stream_tag(p->operand_id, kPurposeSample, 0),
                                                       step, keys); count_launch();
      sample_select_kernel<<<1, 1024, 0, st>>>(keys, r, (int)lk, idx); count_launch();
    } else {
      iota_kernel<<<blocks_for(lk), 256, 0, st>>>(lk, idx); count_launch();
    }
    if (f->sampled_rows)
      cudaMemcpyAsync(f->sampled_rows, idx, (size_t)lk * 4, cudaMemcpyDeviceToDevice, st);
    omega_kernel<<<blocks_for(((int64_t)c * w + 3) / 4), 256, 0, st>>>((int64_t)c * w, p->seed,
                                                                      stream_tag(p->operand_id, kPurposeOmega, 0),
                                                                      step, omega, f->omega); count_launch();
    // Y = M_s Omega ; Q = Y R^+
    if (sampled) {
      rows_times(idx, lk, omega, w, Y);
    } else if ((s = project(omega, w, Y)) != METIS_OK) {
      return s;
    }
    gram(Y, lk, w);
    small_solver_kernel<<<1, 1024, small_smem, st>>>(G, w, k, 0, so, ctx->status); count_launch();
    times_small_kernel<<<blocks_for(lk * w), 256, 0, st>>>(Y, lk, w, T, w, Q); count_launch();
    // Bm^T = M_s^T Q ; R2 = chol(Bm Bm^T) ; SVD(R2^T) ; V = Bm^T R2^+ W'[:, :k]
    cols_times_matrix_kernel<<<blocks_for(c, 64), 256, 0, st>>>(Mb, M->ld, idx, lk, c, Q, w, Bt); count_launch();
    gram(Bt, c, w);
    small_solver_kernel<<<1, 1024, small_smem, st>>>(G, w, k, 1, so, ctx->status); count_launch();
    times_small_kernel<<<blocks_for(c * k), 256, 0, st>>>(Bt, c, w, T, k, f->V); count_launch();
  }
  // per step: P = M V ; R = chol(P^T P) ; SVD(R) ; U = P R^+ U_r ; V <- V V_r
  if ((s = project(f->V, k, Y)) != METIS_OK) return s;
  gram(Y, r, k);
  small_solver_kernel<<<1, 1024, small_smem, st>>>(G, k, k, 2, so, ctx->status); count_launch();
  times_small_kernel<<<blocks_for(r * k), 256, 0, st>>>(Y, r, k, T, k, Q); count_launch();     // U (unsigned)
  times_small_kernel<<<blocks_for(c * k), 256, 0, st>>>(f->V, c, k, Vr, k, Bt); count_launch();  // V V_r
  sign_pick_kernel<<<k, 256, 0, st>>>(Bt, c, k, flip); count_launch();
  apply_flip_kernel<<<blocks_for(c * k), 256, 0, st>>>(Bt, c, k, flip, f->V); count_launch();
  apply_flip_kernel<<<blocks_for(r * k), 256, 0, st>>>(Q, r, k, flip, f->U); count_launch();
  cudaMemcpyAsync(f->S, Sw, (size_t)k * 4, cudaMemcpyDeviceToDevice, st);
  if ((s = check_cuda(ctx, cudaGetLastError(), "decompose")) != METIS_OK) return s;
  // factor quantization (blocks along the long dimension, power-of-two tensor scale)
  float* amax = reinterpret_cast<float*>(flags + 8);
  e = launch_quantize_factor(f->U, r, k, p->rounding, p->seed, p->operand_id, kSrLeft, step, &f->Uq, amax,
                             ctx->status, st);
  if (e != cudaSuccess) return check_cuda(ctx, e, "factor quantization");
  e = launch_quantize_factor(f->V, c, k, p->rounding, p->seed, p->operand_id, kSrRight, step, &f->Vq, amax + 1,
                             ctx->status, st);
  return check_cuda(ctx, e, "factor quantization");
}

}  // namespace metis
