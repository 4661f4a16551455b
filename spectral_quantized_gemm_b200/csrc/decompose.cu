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
// A pair rotates while its off-diagonal cosine |g| / sqrt(a b) exceeds this.  The Gram
// matrices come from products formed with bf16 hi/lo operands on the tensor cores (about
// 16 significant bits), so their entries carry relative errors near 1e-5; rotating further
// only resolves that rounding.  At 1e-5 the eigenvalues are exact to second order and the
// eigenvectors to the Gram's own accuracy, and an operand whose basis already diagonalizes
// its Gram (an unchanged matrix) needs no sweep.
constexpr double kJacobiTol = 1e-5;
// The two-kernel solver also leaves alone an off-diagonal entry below this, in units of
// the largest diagonal entry (it works on the matrix scaled to make that entry 1..2):
// entries at rounding level of a rank-deficient Gram would otherwise keep its
// near-zero eigenvalues rotating among themselves for good, and no eigenvalue above the
// drop threshold (kDropTol) moves by more than (1e-13)^2 / gap.
constexpr double kJacobiFloor = 1e-13;
constexpr int kJacobiMaxSweeps = 40;
constexpr int kMaxW = 128;
constexpr int kSmallMaxN = 96;                 // sketch width limit of the one-CTA solver

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
    if (threadIdx.x < 32) {
      // warp 0 finds the bin where the running count reaches `need`: lane l holds bins
      // 8 l .. 8 l + 7; an inclusive shuffle scan of the lane sums gives each lane the count
      // below its bins, and the lane whose bins cross `need` walks them
      const int l = threadIdx.x;
      unsigned int h[8], sum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        h[t] = hist[8 * l + t];
        sum += h[t];
      }
      unsigned int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (l >= off) incl += v;
      }
      const int64_t nd = need;
      const int64_t below = (int64_t)(incl - sum);
      const bool mine = below < nd && (int64_t)incl >= nd;
      if (mine) {
        int64_t cum = below;
        int b = 8 * l;
        for (int t = 0; t < 8; ++t, ++b) {
          if (cum + h[t] >= nd) break;
          cum += h[t];
        }
        need = nd - cum;
        prefix |= (uint64_t)b << shift;
        mask |= (uint64_t)255u << shift;
      }
    }
    __syncthreads();
  }
  const uint64_t thr = prefix;  // the l_k-th smallest key; keys are distinct
  const int64_t chunk = (rows + blockDim.x - 1) / blockDim.x;
  const int64_t lo = threadIdx.x * chunk, hi = min(rows, lo + chunk);
  int64_t cnt = 0;
  for (int64_t i = lo; i < hi; ++i) cnt += keys[i] <= thr;
  // exclusive block scan of the counts: shuffle scans within warps, then of the warp totals
  {
    const int l = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int64_t incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (l >= off) incl += v;
    }
    if (l == 31) scan[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int64_t tot = l < (int)(blockDim.x >> 5) ? scan[l] : 0;
      int64_t wi = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, wi, off);
        if (l >= off) wi += v;
      }
      scan[32 + l] = wi - tot;   // exclusive prefix of the warp totals
    }
    __syncthreads();
    cnt = scan[32 + wid] + incl - cnt;
  }
  __syncthreads();
  int64_t pos = cnt;
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
// grid: (ceil(nr/64), nsplit), block 256; partial layout [split][nr][w].
// Thread t owns row r = t % 64 and the outputs j = t / 64 + 4 i (registers).
constexpr int kRowsPerBlock = 64;
constexpr int kColChunk = 32;
constexpr int kPerThread = kMaxW / 4;
__global__ void __launch_bounds__(256) rows_times_matrix_kernel(
    const __nv_bfloat16* __restrict__ M, int64_t ld, const int32_t* rowmap, int64_t nr, int64_t ncols,
    const float* __restrict__ B, int w, int64_t split_len, float* __restrict__ partial, uint32_t* status) {
  __shared__ float sm[kRowsPerBlock][kColChunk + 1];
  __shared__ float sb[kColChunk][kMaxW];
  const int64_t r0 = (int64_t)blockIdx.x * kRowsPerBlock;
  const int64_t c_begin = (int64_t)blockIdx.y * split_len;
  const int64_t c_end = min(ncols, c_begin + split_len);
  const int r = threadIdx.x & 63, j0 = threadIdx.x >> 6;
  float acc[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) acc[i] = 0.0f;
  bool finite = true;
  for (int64_t c0 = c_begin; c0 < c_end; c0 += kColChunk) {
    // every load of the chunk in flight before the first shared-memory store
    constexpr int kML = kRowsPerBlock * kColChunk / 256, kBL = kColChunk * kMaxW / 256;
    float mv[kML], bv[kBL];
#pragma unroll
    for (int it = 0; it < kML; ++it) {
      const int e = threadIdx.x + it * 256, rr = e / kColChunk, c = e % kColChunk;
      const int64_t row = r0 + rr;
      float v = 0.0f;
      if (row < nr && c0 + c < c_end) {
        const int64_t src = rowmap ? rowmap[row] : row;
        v = __bfloat162float(M[src * ld + c0 + c]);
      }
      mv[it] = v;
    }
#pragma unroll
    for (int it = 0; it < kBL; ++it) {
      const int e = threadIdx.x + it * 256, c = e / kMaxW, j = e % kMaxW;
      bv[it] = (c0 + c < c_end && j < w) ? B[(c0 + c) * w + j] : 0.0f;
    }
#pragma unroll
    for (int it = 0; it < kML; ++it) {
      const int e = threadIdx.x + it * 256;
      finite &= isfinite(mv[it]);
      sm[e / kColChunk][e % kColChunk] = mv[it];
    }
#pragma unroll
    for (int it = 0; it < kBL; ++it) {
      const int e = threadIdx.x + it * 256;
      sb[e / kMaxW][e % kMaxW] = bv[it];
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kColChunk; ++c) {
      const float a = sm[r][c];
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) acc[i] = fmaf(a, sb[c][j0 + 4 * i], acc[i]);
    }
    __syncthreads();
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  if (r0 + r < nr) {
    float* dst = partial + ((int64_t)blockIdx.y * nr + r0 + r) * w;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i)
      if (j0 + 4 * i < w) dst[j0 + 4 * i] = acc[i];
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
// Thread t owns column c = t % 64 and the outputs j = t / 64 + 4 i (registers).
__global__ void __launch_bounds__(256) cols_times_matrix_kernel(
    const __nv_bfloat16* __restrict__ M, int64_t ld, const int32_t* rowmap, int64_t nr, int64_t ncols,
    const float* __restrict__ Q, int w, float* __restrict__ out) {
  __shared__ float sm[16][65];
  __shared__ float sq[16][kMaxW];
  const int64_t c0 = (int64_t)blockIdx.x * 64;
  const int c = threadIdx.x & 63, j0 = threadIdx.x >> 6;
  float acc[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) acc[i] = 0.0f;
  for (int64_t r0 = 0; r0 < nr; r0 += 16) {
    // every load of the chunk in flight before the first shared-memory store
    float mv[16 * 64 / 256], qv[16 * kMaxW / 256];
#pragma unroll
    for (int it = 0; it < 16 * 64 / 256; ++it) {
      const int e = threadIdx.x + it * 256, rr = e / 64, cc = e % 64;
      float v = 0.0f;
      if (r0 + rr < nr && c0 + cc < ncols) {
        const int64_t src = rowmap ? rowmap[r0 + rr] : r0 + rr;
        v = __bfloat162float(M[src * ld + c0 + cc]);
      }
      mv[it] = v;
    }
#pragma unroll
    for (int it = 0; it < 16 * kMaxW / 256; ++it) {
      const int e = threadIdx.x + it * 256, rr = e / kMaxW, j = e % kMaxW;
      qv[it] = (r0 + rr < nr && j < w) ? Q[(r0 + rr) * w + j] : 0.0f;
    }
#pragma unroll
    for (int it = 0; it < 16 * 64 / 256; ++it) {
      const int e = threadIdx.x + it * 256;
      sm[e / 64][e % 64] = mv[it];
    }
#pragma unroll
    for (int it = 0; it < 16 * kMaxW / 256; ++it) {
      const int e = threadIdx.x + it * 256;
      sq[e / kMaxW][e % kMaxW] = qv[it];
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < 16; ++rr) {
      const float a = sm[rr][c];
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) acc[i] = fmaf(a, sq[rr][j0 + 4 * i], acc[i]);
    }
    __syncthreads();
  }
  if (c0 + c < ncols) {
    float* dst = out + (c0 + c) * w;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i)
      if (j0 + 4 * i < w) dst[j0 + 4 * i] = acc[i];
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
// partial[block] = A_rows^T A_rows over the block's rows, rows staged 32 at a time in
// shared memory as fp64; a thread owns 4 x 4 tiles (ta <= tb) of the upper triangle
// and keeps their 16 sums in registers.  TPT = tiles per thread (1 covers w <= 64).
constexpr int kGramRows = 32;
template <int TPT>
__global__ void __launch_bounds__(256) gram_partial_kernel(const float* __restrict__ A, int64_t n, int w,
                                                           int64_t rows_per_block, double* partial,
                                                           uint32_t* status) {
  __shared__ __align__(16) double sa[kGramRows][kMaxW + 2];
  const int64_t r_begin = (int64_t)blockIdx.x * rows_per_block;
  const int64_t r_end = min(n, r_begin + rows_per_block);
  const int nt = (w + 3) / 4;
  int ta[TPT], tb[TPT];
  double acc[TPT][16];
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    const int t = threadIdx.x + u * 256;
    ta[u] = t / nt;
    tb[u] = t - (t / nt) * nt;
    if (ta[u] >= nt || ta[u] > tb[u]) ta[u] = -1;
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[u][e] = 0.0;
  }
  bool finite = true;
  const int wp = nt * 4;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kGramRows) {
    __syncthreads();
    for (int e = threadIdx.x; e < kGramRows * wp; e += 256) {
      const int r = e / wp, j = e - (e / wp) * wp;
      const float v = (r0 + r < r_end && j < w) ? A[(r0 + r) * w + j] : 0.0f;
      finite &= isfinite(v);
      sa[r][j] = v;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < TPT; ++u) {
      if (ta[u] < 0) continue;
      const double* pa = &sa[0][4 * ta[u]];
      const double* pb = &sa[0][4 * tb[u]];
#pragma unroll 4
      for (int r = 0; r < kGramRows; ++r) {
        const double2 a01 = *reinterpret_cast<const double2*>(pa + r * (kMaxW + 2));
        const double2 a23 = *reinterpret_cast<const double2*>(pa + r * (kMaxW + 2) + 2);
        const double2 b01 = *reinterpret_cast<const double2*>(pb + r * (kMaxW + 2));
        const double2 b23 = *reinterpret_cast<const double2*>(pb + r * (kMaxW + 2) + 2);
        const double av[4] = {a01.x, a01.y, a23.x, a23.y}, bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[u][x * 4 + y] = fma(av[x], bv[y], acc[u][x * 4 + y]);
      }
    }
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  double* out = partial + (int64_t)blockIdx.x * w * w;
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    if (ta[u] < 0) continue;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int a = 4 * ta[u] + x, b = 4 * tb[u] + y;
        if (a < w && b < w && a <= b) out[a * w + b] = acc[u][x * 4 + y];
      }
  }
}

// G (w x w, full) = sum of the blocks' upper triangles, a warp per entry: lane l adds
// blocks l, l + 32, ... in order, then a fixed shuffle tree (deterministic).
__global__ void gram_reduce_kernel(const double* __restrict__ partial, int nblocks, int w, double* __restrict__ G) {
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= w * w) return;
  const int a = e / w, b = e - (e / w) * w;
  const int src = a <= b ? e : b * w + a;
  double acc = 0.0;
  for (int c = lane; c < nblocks; c += 32) acc += partial[(int64_t)c * w * w + src];
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) G[e] = acc;
}

// ----------------------------------------------------- single-CTA small solvers
// Both take the Gram matrix G (n x n, fp64) of a tall matrix Y and run in one CTA of
// a few hundred threads; the problems are a few hundred thousand flops, so the design
// goal is few barrier-separated steps with independent work inside each.
//
// cholqr_solver_kernel (sketches wider than kSmallMaxN, global scratch): T = R^+ with
//   G = R^T R (Cholesky with dependent-column drop), so that Q = Y T is the CholQR factor.  Right-looking on unscaled rows
//   (B_it -= B_ji B_jt / d_j) in panels of kPanel pivots, then R^+ by blocked back
//   substitution on the identity.
// eig_solver_kernel: the SVD of Y through the symmetric eigenproblem of G = Y^T Y =
//   Z Lambda Z^T (two-sided Jacobi, Brent-Luk parallel ordering: a round's disjoint
//   rotations are applied to H as one step over its 2 x 2 blocks), ordered by
//   descending eigenvalue: S = sqrt(lambda), Vr = Z[:, :k] and T = Z[:, :k] Lambda^-1/2,
//   so that Y T are the left singular vectors.  An eigenvalue not above
//   kDropTol * lambda_max counts as zero (zero column of T, zero singular value).
constexpr int kSolverThreads = 256;                 // Cholesky solver
constexpr int kSolverWarps = kSolverThreads / 32;
constexpr int kEigThreads = 1024;                   // eigensolver: a warp per rotation pair
constexpr int kPanel = 8;
constexpr int kLaneRows = (kMaxW + 31) / 32;   // entries of a row or column per lane

struct SmallOut {
  double* T;      // n x kMaxW (row-major, ld kMaxW)
  double* Vr;     // n x kMaxW
  float* S;       // k
  int* flags;     // [0] = numeric failure, [1] = Jacobi sweeps of the last solve
  double* scratch;  // small_solver_doubles(kMaxW), used when the sketch is wider than kSmallMaxN
};

// fp64 words of shared memory (or scratch) either solver uses for a width ne problem
__host__ __device__ constexpr size_t small_solver_doubles(int ne) {
  return (size_t)2 * ne * (ne + 1);
}

__device__ __forceinline__ int rr_index(int pos, int round, int ne) {
  // position 0 stays; positions 1 .. ne-1 rotate by one each round
  if (pos == 0) return 0;
  int v = pos - 1 + round;
  if (v >= ne - 1) v -= ne - 1;
  return v + 1;
}

__device__ __forceinline__ void round_pair(int pr, int round, int ne, int& p, int& q) {
  p = rr_index(pr, round, ne);
  q = rr_index(ne - 1 - pr, round, ne);
  if (p > q) {
    const int t = p;
    p = q;
    q = t;
  }
}

__global__ void __launch_bounds__(kSolverThreads) cholqr_solver_kernel(const double* __restrict__ G, int n,
                                                                       SmallOut out) {
  const int ne = (n + 1) & ~1;
  const int ld = ne;       // R / Cholesky work array, ld x ld
  const int lp = ne + 1;   // odd column stride of the right-hand sides
  double* const bR = out.scratch;
  double* const bV = bR + ld * ld;
  __shared__ int dropped[kMaxW];
  __shared__ double invd[kMaxW];        // 1 / d_j (0 for a dropped pivot)
  __shared__ double rinv[kMaxW];        // 1 / R_jj (0 for a dropped pivot)
  __shared__ double gmax_s;
  const int tid = threadIdx.x;
  const int ty = tid >> 5, tx = tid & 31;
  constexpr int W = kSolverWarps;

  for (int e = tid; e < n * n; e += kSolverThreads) {
    const int i = e / n, j = e - (e / n) * n;
    if (j >= i) bR[i * ld + j] = G[e];
  }
  if (ty == 0) {
    double g = 0.0;
    for (int j = tx; j < n; j += 32) g = fmax(g, G[j * n + j]);
#pragma unroll
    for (int off = 16; off; off >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, off));
    if (tx == 0) gmax_s = g;
  }
  __syncthreads();
  const double tol = kDropTol * gmax_s;

  // ---- Cholesky in panels: warp 0 factors the panel rows, all threads update the rest
  for (int jb = 0; jb < n; jb += kPanel) {
    const int je = min(n, jb + kPanel);
    if (ty == 0) {
      for (int j = jb; j < je; ++j) {
        const double d = bR[j * ld + j];
        const bool drop = !(d > tol) || gmax_s == 0.0;
        const double inv_d = drop ? 0.0 : 1.0 / d;
        if (tx == 0) {
          dropped[j] = drop;
          invd[j] = inv_d;
        }
        if (!drop) {
          for (int i = j + 1; i < je; ++i) {
            const double coef = bR[j * ld + i] * inv_d;
            for (int t = i + tx; t < n; t += 32) bR[i * ld + t] = fma(-coef, bR[j * ld + t], bR[i * ld + t]);
          }
        }
        __syncwarp();
      }
    }
    __syncthreads();
    // trailing rows i >= je: B_it -= sum_j B_ji B_jt / d_j over the panel, t >= i
    const int m = n - je;
    if (m > 0) {
      const int np = je - jb;
      for (int e = tid; e < m * 32; e += kSolverThreads) {
        const int i = je + e / 32, lane = e & 31;
        double cf[kPanel];
#pragma unroll
        for (int q = 0; q < kPanel; ++q) cf[q] = q < np ? bR[(jb + q) * ld + i] * invd[jb + q] : 0.0;
        for (int t = i + lane; t < n; t += 32) {
          double acc = bR[i * ld + t];
#pragma unroll
          for (int q = 0; q < kPanel; ++q)
            if (q < np) acc = fma(-cf[q], bR[(jb + q) * ld + t], acc);
          bR[i * ld + t] = acc;
        }
      }
    }
    __syncthreads();
  }
  for (int j = tid; j < n; j += kSolverThreads) rinv[j] = dropped[j] ? 0.0 : rsqrt(bR[j * ld + j]);
  __syncthreads();
  // R (scaled) column-major into the lower part: R[r][i] at bR[i * ld + r]
  for (int j = ty; j < ne; j += W) {
    for (int t = j + tx; t < ne; t += 32) {
      double v = 0.0;
      if (t < n && j < n && !dropped[j]) v = bR[j * ld + t] * rinv[j];
      bR[t * ld + j] = v;
    }
  }
  // identity right-hand sides, column c at bV + c * lp
  for (int e = tid; e < ne * lp; e += kSolverThreads) {
    const int c = e / lp, r = e - c * lp;
    bV[e] = (c == r && c < n) ? 1.0 : 0.0;
  }
  __syncthreads();

  // ---- blocked back substitution R X = I; x_i = B_i / R_ii (0 for a dropped pivot)
  for (int ie = n; ie > 0; ie -= kPanel) {
    const int ib = max(0, ie - kPanel);
    for (int c = tid; c < n; c += kSolverThreads) {   // diagonal block, a thread per column
      double* col = bV + c * lp;
      for (int i = ie - 1; i >= ib; --i) {
        const double x = col[i] * rinv[i];
        col[i] = x;
        for (int r = ib; r < i; ++r) col[r] = fma(-bR[i * ld + r], x, col[r]);
      }
    }
    __syncthreads();
    if (ib > 0) {   // rows above the block: B_r -= sum_i R[r][i] x_i
      const int nb = ie - ib;
      for (int c = ty; c < n; c += W) {
        double* col = bV + c * lp;
        double x[kPanel];
#pragma unroll
        for (int q = 0; q < kPanel; ++q) x[q] = q < nb ? col[ib + q] : 0.0;
        for (int r = tx; r < ib; r += 32) {
          double acc = col[r];
#pragma unroll
          for (int q = 0; q < kPanel; ++q)
            if (q < nb) acc = fma(-bR[(ib + q) * ld + r], x[q], acc);
          col[r] = acc;
        }
      }
    }
    __syncthreads();
  }
  for (int e = tid; e < n * n; e += kSolverThreads) {
    const int i = e / n, c = e - (e / n) * n;
    out.T[i * kMaxW + c] = bV[c * lp + i];
  }
}

// T = R^+ for G = R^T R (CholQR of a tall Y with G = Y^T Y), n <= kSmallMaxN, one CTA:
// right-looking Cholesky of the lower triangle (G = L L^T, L = R^T) on unscaled columns,
// A_ik -= A_ij A_kj / d_j, two barriers per pivot; a pivot d_j not above
// kDropTol * max diag(G) drops column j (zero row of R, zero column of Q).  Then
// X = L^{-1} by forward substitution on the identity, all columns at once, and
// T = X^T.  A warp per row, lanes along the row: no divisions in the index math.
constexpr int kCholThreads = 512;
__host__ __device__ constexpr size_t chol_smem_bytes(int n) { return (size_t)2 * n * (n + 1) * sizeof(double); }
__global__ void __launch_bounds__(kCholThreads) chol_inverse_kernel(const double* __restrict__ G, int n,
                                                                    SmallOut out) {
  extern __shared__ double smem_d[];
  const int ld = n + 1;
  double* const A = smem_d;            // A[i * ld + k], k <= i
  double* const X = smem_d + n * ld;   // L^{-1}, X[i * ld + c], c <= i
  __shared__ double linv[kMaxW];       // 1 / L_jj = d_j^{-1/2}, 0 for a dropped pivot
  __shared__ double gmax_s;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int W = kCholThreads / 32;
  for (int e = tid; e < n * n; e += kCholThreads) {
    const int i = e / n, k = e - (e / n) * n;
    if (k <= i) A[i * ld + k] = G[e];
    X[i * ld + k] = (i == k) ? 1.0 : 0.0;
  }
  if (warp == 0) {
    double g = 0.0;
    for (int j = lane; j < n; j += 32) g = fmax(g, G[j * n + j]);
#pragma unroll
    for (int off = 16; off; off >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, off));
    if (lane == 0) gmax_s = g;
  }
  __syncthreads();
  const double tol = kDropTol * gmax_s;
  for (int j = 0; j < n; ++j) {
    if (tid == 0) {
      const double d = A[j * ld + j];
      const bool drop = !(d > tol) || gmax_s == 0.0;
      linv[j] = drop ? 0.0 : rsqrt(d);
    }
    __syncthreads();
    const double invd = linv[j] * linv[j];
    if (invd != 0.0) {
      for (int i = j + 1 + warp; i < n; i += W) {
        const double f = A[i * ld + j] * invd;
        for (int k = j + 1 + lane; k <= i; k += 32) A[i * ld + k] = fma(-f, A[k * ld + j], A[i * ld + k]);
      }
    }
    __syncthreads();
  }
  // X = L^{-1}: row i is final once scaled by 1 / L_ii; then rows r > i drop L_ri X_i
  for (int i = 0; i < n; ++i) {
    const double s = linv[i];
    for (int c = tid; c <= i; c += kCholThreads) X[i * ld + c] *= s;
    __syncthreads();
    for (int r = i + 1 + warp; r < n; r += W) {
      const double l = A[r * ld + i] * s;   // L_ri
      if (l != 0.0)
        for (int c = lane; c <= i; c += 32) X[r * ld + c] = fma(-l, X[i * ld + c], X[r * ld + c]);
    }
    __syncthreads();
  }
  for (int e = tid; e < n * n; e += kCholThreads) {
    const int i = e / n, c = e - (e / n) * n;
    out.T[i * kMaxW + c] = (i <= c) ? X[c * ld + i] : 0.0;   // T = X^T (upper triangular)
  }
}

// mode 1: T only (refresh basis); mode 2: T, Vr and S (per-step factors).  Works in global
// scratch; used for sketches wider than the two-kernel solver below takes.
__global__ void __launch_bounds__(kEigThreads) eig_solver_kernel(const double* __restrict__ G, int n, int k,
                                                                    int mode, SmallOut out, uint32_t* status) {
  const int ne = (n + 1) & ~1;
  const int ld = ne + 1;   // odd stride: rows and columns of H, columns of Z, all conflict-free
  double* const H = out.scratch;                     // H[i * ld + j], symmetric
  double* const Z = H + ne * ld;                     // column c at Z + c * ld
  __shared__ double lam[kMaxW];
  __shared__ int order[kMaxW];
  __shared__ double rot_c[kMaxW / 2], rot_s[kMaxW / 2];
  // flags double-buffered by parity: a flag is cleared one step before it is set and
  // read, so no thread clears it while another still reads it
  __shared__ int round_rot[2], need_rot[2];
  const int tid = threadIdx.x;
  const int ty = tid >> 5, tx = tid & 31;
  constexpr int W = kEigThreads / 32;
  constexpr int LR = kLaneRows;   // entries of a row or column per lane

  for (int e = tid; e < ne * ld; e += kEigThreads) {
    const int i = e / ld, j = e - (e / ld) * ld;
    H[e] = (i < n && j < n) ? G[i * n + j] : 0.0;
    Z[e] = (i == j) ? 1.0 : 0.0;
  }
  if (tid == 0) need_rot[0] = 0;
  __syncthreads();
  const int npairs = ne / 2;
  const double tol2 = kJacobiTol * kJacobiTol;
  // A sweep that would rotate no pair ends the iteration; so before each sweep every
  // pair is checked at once (one step instead of a sweep of rounds that rotates nothing).
  int sweep = 0;
  for (; sweep < kJacobiMaxSweeps; ++sweep) {
    {
      bool need = false;
      for (int p = ty; p < ne && !need; p += W)
        for (int q = p + 1 + tx; q < ne; q += 32) {
          const double ga = H[p * ld + q];
          need = need || (ga != 0.0 && ga * ga > tol2 * (H[p * ld + p] * H[q * ld + q]));
        }
      if (need) need_rot[sweep & 1] = 1;
      if (tid == 0) {
        need_rot[(sweep + 1) & 1] = 0;   // last read after the previous sweep's check
        round_rot[0] = 0;                // last read before the previous round's barrier
      }
    }
    __syncthreads();
    if (!need_rot[sweep & 1]) break;
    for (int round = 0; round < ne - 1; ++round) {
      if (tid == 0) round_rot[(round + 1) & 1] = 0;   // last read in round - 1
      // (1) rotation parameters, a thread per pair: with al = H_pp, be = H_qq,
      // ga = H_pq, t = sign(zeta) / (|zeta| + sqrt(1 + zeta^2)), zeta = (be - al) / (2 ga),
      // c = 1 / sqrt(1 + t^2), s = c t (written without divisions)
      for (int pr = tid; pr < npairs; pr += kEigThreads) {
        int p, q;
        round_pair(pr, round, ne, p, q);
        const double al = H[p * ld + p], be = H[q * ld + q], ga = H[p * ld + q];
        double c = 1.0, s = 0.0;
        if (ga != 0.0 && ga * ga > tol2 * (al * be)) {
          const double dd = be - al;
          const double g2 = 2.0 * ga;
          const double x = fma(dd, dd, g2 * g2);
          const double rt = x * rsqrt(x);
          const double den = fabs(dd) + rt;
          const double rho = rsqrt(fma(den, den, g2 * g2));
          const double sgn = (dd == 0.0) ? 1.0 : copysign(1.0, dd) * copysign(1.0, ga);
          c = den * rho;
          s = sgn * fabs(g2) * rho;
          round_rot[round & 1] = 1;
        }
        rot_c[pr] = c;
        rot_s[pr] = s;
      }
      __syncthreads();
      if (round_rot[round & 1]) {   // uniform
        // (2) H <- J^T H J and Z <- Z J with J the round's disjoint rotations: a thread per
        // 2 x 2 block (rows p_i, q_i; columns p_j, q_j), all reads of a block before
        // its writes; a warp per column pair of Z
        for (int e = tid; e < npairs * npairs; e += kEigThreads) {
          const int i = e / npairs, j = e - (e / npairs) * npairs;
          const double si = rot_s[i], sj = rot_s[j];
          if (si == 0.0 && sj == 0.0) continue;
          const double ci = rot_c[i], cj = rot_c[j];
          int pa, pb, qa, qb;
          round_pair(i, round, ne, pa, pb);
          round_pair(j, round, ne, qa, qb);
          const double h00 = H[pa * ld + qa], h01 = H[pa * ld + qb];
          const double h10 = H[pb * ld + qa], h11 = H[pb * ld + qb];
          const double r00 = ci * h00 - si * h10, r10 = si * h00 + ci * h10;   // rows
          const double r01 = ci * h01 - si * h11, r11 = si * h01 + ci * h11;
          H[pa * ld + qa] = cj * r00 - sj * r01;                                 // columns
          H[pa * ld + qb] = sj * r00 + cj * r01;
          H[pb * ld + qa] = cj * r10 - sj * r11;
          H[pb * ld + qb] = sj * r10 + cj * r11;
        }
        for (int pr = ty; pr < npairs; pr += W) {
          const double s = rot_s[pr];
          if (s == 0.0) continue;
          const double c = rot_c[pr];
          int p, q;
          round_pair(pr, round, ne, p, q);
          double* zp = Z + p * ld;
          double* zq = Z + q * ld;
          double za[LR], zb[LR];
#pragma unroll
          for (int u = 0; u < LR; ++u) {
            const int x = tx + 32 * u;
            if (x < ne) {
              za[u] = zp[x];
              zb[u] = zq[x];
            }
          }
#pragma unroll
          for (int u = 0; u < LR; ++u) {
            const int x = tx + 32 * u;
            if (x < ne) {
              zp[x] = c * za[u] - s * zb[u];
              zq[x] = s * za[u] + c * zb[u];
            }
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    out.flags[1] = sweep;   // sweeps taken (diagnostic)
    if (sweep == kJacobiMaxSweeps) {
      raise_status(status, METIS_DEV_NUMERIC);
      out.flags[0] = 1;
    }
  }
  // eigenvalues and descending order (ties by index; a NaN sorts last)
  for (int j = tid; j < ne; j += kEigThreads) {
    const double l = H[j * ld + j];
    lam[j] = (l == l) ? l : -HUGE_VAL;
  }
  __syncthreads();
  for (int j = tid; j < ne; j += kEigThreads) {
    int rank = 0;
    for (int i = 0; i < ne; ++i) rank += (lam[i] > lam[j]) || (lam[i] == lam[j] && i < j);
    order[rank] = j;
  }
  __syncthreads();
  const double lmax = fmax(lam[order[0]], 0.0);
  const double thr = kDropTol * lmax;
  for (int e = tid; e < n * k; e += kEigThreads) {
    const int i = e / k, c = e - (e / k) * k;
    const int src = order[c];
    const double l = lam[src];
    const bool keep = l > thr && lmax > 0.0;
    const double z = Z[src * ld + i];
    out.T[i * kMaxW + c] = keep ? z * rsqrt(l) : 0.0;
    if (mode == 2) out.Vr[i * kMaxW + c] = z;
  }
  if (mode == 2) {
    for (int c = tid; c < k; c += kEigThreads) {
      const double l = lam[order[c]];
      out.S[c] = (l > thr && lmax > 0.0) ? (float)sqrt(l) : 0.0f;
    }
  }
}

// ------------------------------------------- two-kernel Jacobi eigensolver (ne <= 88)
// The eigenproblem of G (n x n, fp64) by cyclic two-sided Jacobi in the round-robin
// (circle) ordering, split in two launches:
//
// jacobi_rounds_kernel (one CTA): the matrix is kept in slot order -- slot pair a =
//   (2a, 2a+1) is the rotation pair of the current round -- and after each round every
//   element moves to its next slot (jac_dest), written into the other of two shared-memory
//   buffers.  Only the upper triangle is kept; a thread owns one 2 x 2 block (a <= b) of
//   the slot grid.  The rotation of the NEXT round's pair a' is computed in the same step
//   by the owner of the block that holds that pair's off-diagonal element; the two new
//   diagonal entries it needs are recomputed from the old diagonal blocks with the same
//   correctly rounded arithmetic the diagonal owners use.  One barrier per round.  The
//   matrix is held scaled by a power of two; entries below kJacobiFloor of it are left.  Each
//   round's rotations (c, s) go to global memory; after a whole number of sweeps every
//   element is back in its own slot, so the diagonal is the spectrum in index order.
// jacobi_replay_kernel (a warp per row of Z): applies the recorded rotations and slot
//   moves to one row of the identity, giving the eigenvector matrix row by row, and
//   writes T = Z Lambda^-1/2 and Vr = Z in descending eigenvalue order.
constexpr int kJacMaxNE = 88;          // m(m - 1)/2 off-diagonal blocks fit in 32 - ceil(m/32) warps, m = ne/2
constexpr int kJacThreads = 1024;
constexpr int kJacChunk = 16;          // replay: rounds of rotations staged per chunk
constexpr int kJacRowsPerCta = 4;      // replay: rows (warps) per CTA

__host__ __device__ constexpr int jac_ne(int n) { return n < 4 ? 4 : (n + 1) & ~1; }
__host__ __device__ constexpr size_t jac_rot_entries(int n) {
  return ((size_t)kJacobiMaxSweeps * (jac_ne(n) - 1) + 1) * (jac_ne(n) / 2);
}
__host__ __device__ constexpr size_t jac_smem_bytes(int ne) {
  return (size_t)2 * ne * ne * sizeof(double) + (size_t)2 * (ne / 2) * (2 * sizeof(double2) + sizeof(double));
}

// slot an element moves to after a round: top of pair 0 stays; the other 2m - 1 slots
// form a ring top_1 -> top_2 -> ... -> top_{m-1} -> bot_{m-1} -> ... -> bot_0 -> top_1
__device__ __forceinline__ int jac_dest(int s, int m) {
  if (s == 0) return 0;
  const int a = s >> 1;
  if ((s & 1) == 0) return a <= m - 2 ? 2 * (a + 1) : 2 * m - 1;
  return a >= 1 ? 2 * a - 1 : 2;
}
__device__ __forceinline__ int jac_src(int s, int m) {
  if (s == 0) return 0;
  const int a = s >> 1;
  if ((s & 1) == 0) return a == 1 ? 1 : 2 * a - 2;
  return a == m - 1 ? 2 * m - 2 : 2 * a + 3;
}

// Whether the two-kernel solver still rotates an entry g between diagonal entries a and b
// (of the scaled matrix).
__device__ __forceinline__ bool jac_needs(double g, double a, double b, double tol2) {
  return g != 0.0 && g * g > tol2 * (a * b) && g * g > kJacobiFloor * kJacobiFloor;
}

// rotation (c, s) that annihilates ga in [[al, ga], [ga, be]] (x_p' = c x_p - s x_q,
// x_q' = s x_p + c x_q), or the identity when jac_needs says no
__device__ __forceinline__ double2 jac_rotation(double al, double be, double ga, double tol2) {
  double c = 1.0, s = 0.0;
  if (jac_needs(ga, al, be, tol2)) {
    const double dd = be - al;
    const double g2 = 2.0 * ga;
    const double x = fma(dd, dd, g2 * g2);
    const double rt = x * rsqrt(x);
    const double den = fabs(dd) + rt;
    const double rho = rsqrt(fma(den, den, g2 * g2));
    const double sgn = (dd == 0.0) ? 1.0 : copysign(1.0, dd) * copysign(1.0, ga);
    c = den * rho;
    s = sgn * fabs(g2) * rho;
  }
  return make_double2(c, s);
}

// new diagonal of a rotated pair; correctly rounded operations only, so every thread
// that evaluates it for the same pair gets the same bits
__device__ __forceinline__ void jac_diag(double al, double be, double ga, double2 cs, double& d0, double& d1) {
  const double cc = __dmul_rn(cs.x, cs.x), ss = __dmul_rn(cs.y, cs.y);
  const double x = __dmul_rn(__dmul_rn(__dmul_rn(2.0, cs.x), cs.y), ga);
  d0 = __fma_rn(cc, al, __fma_rn(ss, be, -x));
  d1 = __fma_rn(ss, al, __fma_rn(cc, be, x));
}

struct JacOut {
  double2* rot;      // jac_rot_entries(n) rotations, round-major
  int* info;         // [0] rounds recorded
  int* order;        // k source slots, descending eigenvalue
  double* inv_sqrt;  // k factors lambda^-1/2 (0 for a dropped eigenvalue)
};

__global__ void __launch_bounds__(kJacThreads, 1) jacobi_rounds_kernel(const double* __restrict__ G, int n, int k,
                                                                       int mode, JacOut jo, SmallOut out,
                                                                       uint32_t* status, int max_sweeps) {
  extern __shared__ double smem_d[];
  const int ne = jac_ne(n), m = ne / 2;
  double* Hbuf0 = smem_d;                       // off-diagonal blocks of the slot grid, upper triangle
  double* Hbuf1 = smem_d + ne * ne;
  double2* prm = reinterpret_cast<double2*>(smem_d + 2 * ne * ne);   // [2][m] rotation (c, s) of pair p
  double2* dgn = prm + 2 * m;                                          // [2][m] diagonal (al, be) of pair p
  double* dof = reinterpret_cast<double*>(dgn + 2 * m);               // [2][m] off-diagonal ga of pair p
  __shared__ double lam[kJacMaxNE];
  __shared__ int order[kJacMaxNE];
  __shared__ double scale_s[2];
  const int tid = threadIdx.x;
  const double tol2 = kJacobiTol * kJacobiTol;

  // The matrix is held scaled by 2^-E (exact), E = floor(log2) of its largest diagonal
  // entry, so that kJacobiFloor is relative to it; the eigenvalues are scaled back.
  if (tid < 32) {
    double g = 0.0;
    for (int j = tid; j < n; j += 32) g = fmax(g, fabs(G[j * n + j]));
#pragma unroll
    for (int off = 16; off; off >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, off));
    if (tid == 0) {
      const bool ok = g > 0.0 && g <= 1.7976931348623157e308;
      const int e = ok ? max(-1000, min(1000, ilogb(g))) : 0;
      scale_s[0] = ldexp(1.0, -e);
      scale_s[1] = ldexp(1.0, e);
    }
  }
  __syncthreads();
  const double down = scale_s[0];
  for (int e = tid; e < ne * ne; e += kJacThreads) {
    const int i = e / ne, j = e - (e / ne) * ne;
    Hbuf0[e] = (i < n && j < n && i <= j) ? G[i * n + j] * down : 0.0;
  }
  // Roles, warp-aligned so that each warp runs one instruction stream.  The pair warps
  // (ceil(m / 32) of them, warps 0, 4, ...) own pair p: its 2 x 2 diagonal block, kept in
  // dgn/dof, and the rotation of the next round's pair p -- the chain that bounds a round --
  // so they sit on the SM sub-partition of warps 0 mod 4, which the block warps fill last.
  // The block warps own the off-diagonal blocks (a < b), warps not 0 mod 4 first.
  const int warp = tid >> 5, lane = tid & 31;
  const int n_pair_warps = (m + 31) / 32;
  const bool pair_warp = (warp & 3) == 0 && (warp >> 2) < n_pair_warps;
  int off_rank;   // position of this warp among the block warps
  if ((warp & 3) != 0) off_rank = warp - (warp >> 2) - 1;
  else off_rank = 24 + (warp >> 2) - n_pair_warps;
  const int n_off = m * (m - 1) / 2;
  const int e_off = off_rank * 32 + lane;
  const bool is_off = !pair_warp && e_off < n_off;
  const int p = pair_warp ? (warp >> 2) * 32 + lane : -1;
  const bool is_pair = pair_warp && p < m;
  int a = 0, b = 0;
  int wr[4] = {0, 0, 0, 0};
  int lo = 0, hi = 0, su = 0, sv = 0, x = 0, y = 0;
  if (is_off) {
    int rem = e_off;
    while (rem >= m - 1 - a) {
      rem -= m - 1 - a;
      ++a;
    }
    b = a + 1 + rem;
    const int da0 = jac_dest(2 * a, m), da1 = jac_dest(2 * a + 1, m);
    const int db0 = jac_dest(2 * b, m), db1 = jac_dest(2 * b + 1, m);
    wr[0] = min(da0, db0) * ne + max(da0, db0);
    wr[1] = min(da0, db1) * ne + max(da0, db1);
    wr[2] = min(da1, db0) * ne + max(da1, db0);
    wr[3] = min(da1, db1) * ne + max(da1, db1);
  } else if (is_pair) {
    const int d0 = jac_dest(2 * p, m), d1 = jac_dest(2 * p + 1, m);
    wr[0] = min(d0, d1) * ne + max(d0, d1);   // where this pair's off-diagonal element goes
    // the next round's pair p is (su, sv) in the current slots; its off-diagonal element
    // lies in block (lo, hi), at (x, y) within it
    su = jac_src(2 * p, m);
    sv = jac_src(2 * p + 1, m);
    const bool fwd = (su >> 1) < (sv >> 1);
    lo = fwd ? su >> 1 : sv >> 1;
    hi = fwd ? sv >> 1 : su >> 1;
    x = fwd ? su & 1 : sv & 1;
    y = fwd ? sv & 1 : su & 1;
  }
  __syncthreads();
  double own_ga = 0.0;
  double2 own_cs = make_double2(1.0, 0.0);
  if (is_pair) {
    const double al = Hbuf0[2 * p * ne + 2 * p], be = Hbuf0[(2 * p + 1) * ne + 2 * p + 1];
    own_ga = Hbuf0[2 * p * ne + 2 * p + 1];
    own_cs = jac_rotation(al, be, own_ga, tol2);
    prm[p] = own_cs;
    dgn[p] = make_double2(al, be);
    dof[p] = own_ga;
    jo.rot[p] = own_cs;
  }
  const double* Hr = Hbuf0;
  double* Hw = Hbuf1;
  int round = 0, sweep = 0;
  for (;; ++sweep) {
    // converged when no pair of the current matrix would rotate
    const double2* Dc = dgn + (round & 1) * m;
    bool need = false;
    if (is_off) {
      const double2 da = Dc[a], db = Dc[b];
      const double h00 = Hr[2 * a * ne + 2 * b], h01 = Hr[2 * a * ne + 2 * b + 1];
      const double h10 = Hr[(2 * a + 1) * ne + 2 * b], h11 = Hr[(2 * a + 1) * ne + 2 * b + 1];
      need = jac_needs(h00, da.x, db.x, tol2) || jac_needs(h01, da.x, db.y, tol2) ||
             jac_needs(h10, da.y, db.x, tol2) || jac_needs(h11, da.y, db.y, tol2);
    } else if (is_pair) {
      const double2 d = Dc[p];
      need = jac_needs(own_ga, d.x, d.y, tol2);
    }
    if (!__syncthreads_or(need)) break;
    if (sweep == max_sweeps) {
      if (tid == 0) {
        raise_status(status, METIS_DEV_NUMERIC);
        out.flags[0] = 1;
      }
      break;
    }
    for (int r = 0; r < ne - 1; ++r, ++round) {
      const int cur = (round & 1) * m, nxt = m - cur;
      if (is_off) {
        const double2 ca = prm[cur + a], cb = prm[cur + b];
        const double2 top = *reinterpret_cast<const double2*>(Hr + 2 * a * ne + 2 * b);
        const double2 bot = *reinterpret_cast<const double2*>(Hr + (2 * a + 1) * ne + 2 * b);
        const double r00 = ca.x * top.x - ca.y * bot.x, r10 = ca.y * top.x + ca.x * bot.x;
        const double r01 = ca.x * top.y - ca.y * bot.y, r11 = ca.y * top.y + ca.x * bot.y;
        Hw[wr[0]] = cb.x * r00 - cb.y * r01;
        Hw[wr[1]] = cb.y * r00 + cb.x * r01;
        Hw[wr[2]] = cb.x * r10 - cb.y * r11;
        Hw[wr[3]] = cb.y * r10 + cb.x * r11;
      } else if (is_pair) {
        const int pu = su >> 1, pv = sv >> 1;
        const double2 ru = *reinterpret_cast<const double2*>(Hr + (2 * lo + x) * ne + 2 * hi);
        const double2 rl = *reinterpret_cast<const double2*>(Hr + (2 * lo + 1 - x) * ne + 2 * hi);
        const double2 clo = prm[cur + lo], chi = prm[cur + hi], cu = prm[cur + pu], cv = prm[cur + pv];
        const double2 du = dgn[cur + pu], dv = dgn[cur + pv];
        const double gu = dof[cur + pu], gv = dof[cur + pv];
        // this pair's own off-diagonal element: annihilated when it rotates
        Hw[wr[0]] = (own_cs.y != 0.0) ? 0.0 : own_ga;
        // next round's pair p: new diagonal entries of its two slots and its rotated
        // off-diagonal element; rotated row x = c (row x) -+ s (other row), minus for the top
        double u0, u1, v0, v1;
        jac_diag(du.x, du.y, gu, cu, u0, u1);
        jac_diag(dv.x, dv.y, gv, cv, v0, v1);
        const double gx = x ? clo.y : -clo.y;
        const double q0 = clo.x * ru.x + gx * rl.x, q1 = clo.x * ru.y + gx * rl.y;   // columns 2hi, 2hi + 1
        own_ga = y ? (chi.y * q0 + chi.x * q1) : (chi.x * q0 - chi.y * q1);
        const double nal = (su & 1) ? u1 : u0, nbe = (sv & 1) ? v1 : v0;
        own_cs = jac_rotation(nal, nbe, own_ga, tol2);
        prm[nxt + p] = own_cs;
        dgn[nxt + p] = make_double2(nal, nbe);
        dof[nxt + p] = own_ga;
        jo.rot[(size_t)(round + 1) * m + p] = own_cs;
      }
      __syncthreads();
      const double* t = Hr;
      Hr = Hw;
      Hw = const_cast<double*>(t);
    }
  }
  // after whole sweeps every element is in its own slot: the diagonal is the spectrum
  const double up = scale_s[1];
  const double2* Dc = dgn + (round & 1) * m;
  for (int j = tid; j < ne; j += kJacThreads) {
    const double l = ((j & 1) ? Dc[j >> 1].y : Dc[j >> 1].x) * up;
    lam[j] = (l == l) ? l : -HUGE_VAL;
  }
  __syncthreads();
  for (int j = tid; j < ne; j += kJacThreads) {
    int rank = 0;
    for (int i = 0; i < ne; ++i) rank += (lam[i] > lam[j]) || (lam[i] == lam[j] && i < j);
    order[rank] = j;
  }
  __syncthreads();
  const double lmax = fmax(lam[order[0]], 0.0);
  const double thr = kDropTol * lmax;
  for (int c = tid; c < k; c += kJacThreads) {
    const double l = lam[order[c]];
    const bool keep = l > thr && lmax > 0.0;
    jo.order[c] = order[c];
    jo.inv_sqrt[c] = keep ? rsqrt(l) : 0.0;
    if (mode == 2) out.S[c] = keep ? (float)sqrt(l) : 0.0f;
  }
  if (tid == 0) {
    jo.info[0] = round;
    out.flags[1] = sweep;
  }
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// One warp per row of Z.  Lane l holds the row's entries at the slots of pairs l and
// l + 32; a round rotates each pair and moves every entry one step along the slot ring
// (two shuffles per set of pairs).  The recorded rotations are staged through shared
// memory in chunks of kJacChunk rounds, the next chunk copied while this one is applied.
__global__ void __launch_bounds__(32 * kJacRowsPerCta) jacobi_replay_kernel(const double2* __restrict__ rot,
                                                                            const int* __restrict__ info, int n,
                                                                            int k, int mode,
                                                                            const int* __restrict__ order,
                                                                            const double* __restrict__ inv_sqrt,
                                                                            SmallOut out) {
  __shared__ __align__(16) double2 chunk[2][kJacChunk * (kJacMaxNE / 2)];
  __shared__ double zrow[kJacRowsPerCta][kJacMaxNE];
  constexpr unsigned kFull = 0xffffffffu;
  const int ne = jac_ne(n), m = ne / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kJacRowsPerCta + warp;
  const int rounds = info[0];
  const int a0 = lane, a1 = lane + 32;
  double t0 = (2 * a0 == row) ? 1.0 : 0.0, b0 = (2 * a0 + 1 == row) ? 1.0 : 0.0;
  double t1 = (2 * a1 == row) ? 1.0 : 0.0, b1 = (2 * a1 + 1 == row) ? 1.0 : 0.0;
  const int nchunks = (rounds + kJacChunk - 1) / kJacChunk;
  auto stage = [&](int ch) {
    const int r0 = ch * kJacChunk;
    const int cnt = (min(rounds, r0 + kJacChunk) - r0) * m;
    double2* dst = chunk[ch & 1];
    const double2* src = rot + (size_t)r0 * m;
    for (int e = threadIdx.x; e < cnt; e += blockDim.x) cp_async16(dst + e, src + e);
    cp_async_commit();
  };
  if (nchunks > 0) stage(0);
  for (int ch = 0; ch < nchunks; ++ch) {
    cp_async_wait_all();
    __syncthreads();                       // chunk ch visible; chunk ch - 1 no longer read
    if (ch + 1 < nchunks) stage(ch + 1);
    const double2* cr = chunk[ch & 1];
    const int nr = min(rounds, (ch + 1) * kJacChunk) - ch * kJacChunk;
    for (int rr = 0; rr < nr; ++rr, cr += m) {
      const double2 c0 = a0 < m ? cr[a0] : make_double2(1.0, 0.0);
      const double2 c1 = a1 < m ? cr[a1] : make_double2(1.0, 0.0);
      const double rt0 = c0.x * t0 - c0.y * b0, rb0 = c0.y * t0 + c0.x * b0;
      const double rt1 = c1.x * t1 - c1.y * b1, rb1 = c1.y * t1 + c1.x * b1;
      // new top[a] = a == 0 ? top[0] : a == 1 ? bot[0] : top[a - 1]
      // new bot[a] = a == m - 1 ? top[m - 1] : bot[a + 1]
      const double up_t0 = __shfl_up_sync(kFull, rt0, 1);
      const double dn_b0 = __shfl_down_sync(kFull, rb0, 1);
      const double bot_0 = __shfl_sync(kFull, rb0, 0);
      double up_t1 = 0.0, dn_b1 = 0.0, w_t0 = 0.0, w_b1 = 0.0;
      if (m > 32) {
        up_t1 = __shfl_up_sync(kFull, rt1, 1);
        dn_b1 = __shfl_down_sync(kFull, rb1, 1);
        w_t0 = __shfl_sync(kFull, rt0, 31);
        w_b1 = __shfl_sync(kFull, rb1, 0);
      }
      t0 = lane == 0 ? rt0 : (lane == 1 ? bot_0 : up_t0);
      b0 = a0 == m - 1 ? rt0 : (lane == 31 ? w_b1 : dn_b0);
      t1 = lane == 0 ? w_t0 : up_t1;
      b1 = a1 == m - 1 ? rt1 : dn_b1;
    }
  }
  if (a0 < m) {
    zrow[warp][2 * a0] = t0;
    zrow[warp][2 * a0 + 1] = b0;
  }
  if (a1 < m) {
    zrow[warp][2 * a1] = t1;
    zrow[warp][2 * a1 + 1] = b1;
  }
  __syncwarp();
  if (row < n) {
    for (int c = lane; c < k; c += 32) {
      const double z = zrow[warp][order[c]];
      out.T[row * kMaxW + c] = z * inv_sqrt[c];
      if (mode == 2) out.Vr[row * kMaxW + c] = z;
    }
  }
}

// ------------------------------------------- tensor-core projection helpers
// out (2kp x n, bf16 row-major): row j < k = hi(F[:, j]), row kp + j = lo(F[:, j]) with
// hi = bf16(F), lo = bf16(F - hi); other rows zero.  F is n x k fp32 row-major.
// A block transposes 64 rows of F (k <= kp <= 128) through shared memory: the rows are read
// whole and each output row j gets 64 consecutive entries, so reads and writes coalesce.
// Every load of a thread is issued before the first shared-memory store (one memory
// round trip per block, not one per element).
constexpr int kSplitRows = 64;
constexpr int kSplitThreads = 512;
__global__ void __launch_bounds__(kSplitThreads) split_hi_lo_t_kernel(const float* __restrict__ F, int64_t n, int k,
                                                                      int kp, __nv_bfloat16* __restrict__ out) {
  __shared__ float t[kSplitRows][129];
  const int64_t i0 = (int64_t)blockIdx.x * kSplitRows;
  const int lkp = __ffs(kp) - 1;   // kp is a power of two
  float v[kSplitRows * 128 / kSplitThreads];
#pragma unroll
  for (int it = 0; it < kSplitRows * 128 / kSplitThreads; ++it) {
    const int e = threadIdx.x + it * kSplitThreads;
    const int r = e >> lkp, c = e & (kp - 1);
    v[it] = (r < kSplitRows && c < k && i0 + r < n) ? F[(i0 + r) * k + c] : 0.0f;
  }
#pragma unroll
  for (int it = 0; it < kSplitRows * 128 / kSplitThreads; ++it) {
    const int e = threadIdx.x + it * kSplitThreads;
    if ((e >> lkp) < kSplitRows) t[e >> lkp][e & (kp - 1)] = v[it];
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < kSplitRows * 128 / kSplitThreads; ++it) {
    const int e = threadIdx.x + it * kSplitThreads;
    const int j = e / kSplitRows, r = e % kSplitRows;
    if (j >= kp || i0 + r >= n) continue;
    const float f = t[r][j];
    const __nv_bfloat16 hi = __float2bfloat16_rn(f);
    out[(int64_t)j * n + i0 + r] = hi;
    out[(int64_t)(kp + j) * n + i0 + r] = __float2bfloat16_rn(f - __bfloat162float(hi));
  }
}

// out (rows x k) = sum over the splits of (hi part + lo part), in split order; the loads
// of four splits go out together
constexpr int kMaxProjSplits = 16;
__global__ void reduce_hi_lo_kernel(const float* __restrict__ partial, int splits, int64_t rows, int kp, int k,
                                    float* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= rows * k) return;
  const int64_t i = e / k;
  const int j = (int)(e - i * k);
  const int64_t stride = rows * 2 * kp;
  const float* row = partial + i * 2 * kp + j;
  float a = 0.0f;
  for (int s0 = 0; s0 < splits; s0 += 4) {
    float h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      h[u] = s0 + u < splits ? row[(s0 + u) * stride] : 0.0f;
      l[u] = s0 + u < splits ? row[(s0 + u) * stride + kp] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < splits) a += h[u] + l[u];
  }
  out[e] = a;
}

int pad_width(int w) { return w <= 16 ? 16 : w <= 32 ? 32 : w <= 64 ? 64 : 128; }

// ---------------------------------------------------- per-step factor finalization
// Counters gathered while the new factors are formed (zeroed before): the largest |.| of
// U and of V (float bits; order-independent atomicMax), and per column j of V V_r the key
// (|v| bits << 32 | ~row) of its largest-|.| entry, first row on ties.
struct FactorStats {
  unsigned long long* amax;   // [0] U, [1] V
  unsigned long long* key;    // k
};

// Uraw (r x k) = P T and Vn (c x k) = V Vr, T and Vr fp64 (ld kMaxW), k <= 64.  A block
// owns 64 rows of one product: the k x k matrix (fp64) and the rows (fp32) are staged in
// shared memory, and each thread forms a 4 x 4 tile of outputs in fp64 (6 loads per 16
// fused multiply-adds).
constexpr int kFpRows = 64;
constexpr size_t kFpSmem = (size_t)64 * 64 * 8 + (size_t)kFpRows * 64 * 4 * 2;
__global__ void __launch_bounds__(256) factor_products_kernel(const float* __restrict__ P, int64_t r,
                                                              const double* __restrict__ T,
                                                              const float* __restrict__ V, int64_t c,
                                                              const double* __restrict__ Vr, int k,
                                                              float* __restrict__ Uraw, float* __restrict__ Vn,
                                                              FactorStats fs, uint32_t* status) {
  extern __shared__ __align__(16) uint8_t fp_smem[];
  double* sm = reinterpret_cast<double*>(fp_smem);                  // [64][64]
  float* sr = reinterpret_cast<float*>(fp_smem + 64 * 64 * 8);      // [kFpRows][64]
  float* so = sr + kFpRows * 64;                                      // [kFpRows][64]
  const int64_t nbu = (r + kFpRows - 1) / kFpRows;
  const bool is_u = blockIdx.x < nbu;
  const int64_t i0 = (int64_t)(is_u ? blockIdx.x : blockIdx.x - nbu) * kFpRows;
  const int64_t n = is_u ? r : c;
  const float* src = is_u ? P : V;
  const double* M = is_u ? T : Vr;
  float* dst = is_u ? Uraw : Vn;
  {
    // all 32 loads of a thread in flight at once, then the shared-memory stores
    double mv[64 * 64 / 256];
    float rv[kFpRows * 64 / 256];
#pragma unroll
    for (int it = 0; it < 64 * 64 / 256; ++it) {
      const int e = threadIdx.x + it * 256, u = e >> 6, j = e & 63;
      mv[it] = (u < k && j < k) ? M[u * kMaxW + j] : 0.0;
    }
#pragma unroll
    for (int it = 0; it < kFpRows * 64 / 256; ++it) {
      const int e = threadIdx.x + it * 256, rr = e >> 6, j = e & 63;
      rv[it] = (i0 + rr < n && j < k) ? src[(i0 + rr) * k + j] : 0.0f;
    }
#pragma unroll
    for (int it = 0; it < 64 * 64 / 256; ++it) sm[threadIdx.x + it * 256] = mv[it];
#pragma unroll
    for (int it = 0; it < kFpRows * 64 / 256; ++it) sr[threadIdx.x + it * 256] = rv[it];
  }
  __syncthreads();
  const int rg = threadIdx.x >> 4, cg = threadIdx.x & 15;   // rows 4 rg .. +3, columns 4 cg .. +3
  double acc[4][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = 0.0;
  for (int u = 0; u < k; ++u) {
    const double2 b01 = *reinterpret_cast<const double2*>(sm + u * 64 + 4 * cg);
    const double2 b23 = *reinterpret_cast<const double2*>(sm + u * 64 + 4 * cg + 2);
    const double bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const double a = (double)sr[(4 * rg + x) * 64 + u];
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = fma(a, bv[y], acc[x][y]);
    }
  }
  float amax = 0.0f;
  bool finite = true;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int64_t i = i0 + 4 * rg + x;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = 4 * cg + y;
      const float v = (float)acc[x][y];
      so[(4 * rg + x) * 64 + j] = v;
      if (i < n && j < k) {
        dst[i * k + j] = v;
        finite &= isfinite(v);
        amax = fmaxf(amax, fabsf(v));
      }
    }
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  // one atomic per block (a warp's maximum, then the block's)
  __shared__ float wmax[8];
#pragma unroll
  for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = wmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    atomicMax(&fs.amax[is_u ? 0 : 1], (unsigned long long)__float_as_uint(m));
  }
  if (!is_u) {
    // the key of each column's largest-|.| entry: four threads per column, 16 rows each
    const int j = threadIdx.x & 63, part = threadIdx.x >> 6;
    if (j < k) {
      unsigned long long best = 0;
      for (int q = part * (kFpRows / 4); q < (part + 1) * (kFpRows / 4) && i0 + q < n; ++q) {
        const float a = fabsf(so[q * 64 + j]);
        if (!(a <= 3.402823466e38f)) continue;   // not finite
        const unsigned long long key =
            ((unsigned long long)__float_as_uint(a) << 32) | (0xFFFFFFFFu - (uint32_t)(i0 + q));
        best = key > best ? key : best;
      }
      if (best) atomicMax(&fs.key[j], best);
    }
  }
}

// U, V (fp32 caller state) = the products with the sign convention applied (column j
// flipped when the largest-|.| entry of Vn's column j is negative), and their NVFP4
// copies: the transposes, blocks of 16 along the long dimension, outer padded to 128 with
// zeros, tensor scale pow2_ceil(max / 2688).  A thread per (16-row block, column < 128).
__global__ void __launch_bounds__(256) factor_finalize_kernel(const float* __restrict__ Uraw, int64_t r,
                                                              const float* __restrict__ Vn, int64_t c, int k,
                                                              FactorStats fs, int rounding, uint64_t seed,
                                                              uint32_t tag_u, uint32_t tag_v, uint32_t step,
                                                              float* __restrict__ U, float* __restrict__ V,
                                                              metis_nvfp4 uq, metis_nvfp4 vq) {
  const int64_t nu = 128 * (r / 16);
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nu + 128 * (c / 16)) return;
  const bool is_u = idx < nu;
  const int64_t t = is_u ? idx : idx - nu;
  const int j = (int)(t & 127);
  const int64_t b = t >> 7;
  const int64_t len = is_u ? r : c;
  const metis_nvfp4& q = is_u ? uq : vq;
  const float g = pow2_ceil(__fdiv_rn(__uint_as_float((uint32_t)fs.amax[is_u ? 0 : 1]), 2688.0f));
  if (t == 0) *q.tensor_scale = g;
  uint2 packed = make_uint2(0, 0);
  uint32_t code = 0;
  if (j < k) {
    const unsigned long long key = fs.key[j];   // 0 only when the column has no finite entry
    const int64_t pivot = key ? (int64_t)(0xFFFFFFFFu - (uint32_t)key) : 0;
    const bool flip = pivot < c && Vn[pivot * k + j] < 0.0f;
    const float* src = is_u ? Uraw : Vn;
    float* dst = is_u ? U : V;
    float v[16];
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float x = src[(b * 16 + e) * k + j];
      v[e] = flip ? -x : x;
      dst[(b * 16 + e) * k + j] = v[e];
      amax = fmaxf(amax, fabsf(v[e]));
    }
    const BlockScale bs = block_scale(amax, g);
    float x[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = __fmul_rn(v[e], bs.rcp);
    packed = encode_block16(x, rounding, seed, is_u ? tag_u : tag_v, step, (uint64_t)j * (uint64_t)len + b * 16);
    if (bs.code == 0) packed = make_uint2(0, 0);
    code = bs.code;
  }
  *reinterpret_cast<uint2*>(q.codes + j * (len / 2) + b * 8) = packed;
  q.scales[scale_offset(j, b, len / 64)] = (uint8_t)code;
}

// Mt (c x r, bf16, row-major) = M^T for M (r x c, leading dimension ld), r and c multiples
// of 64: 64 x 64 tiles through shared memory, rows read and written as 128-byte lines.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ M, int64_t ld,
                                                             int64_t r, __nv_bfloat16* __restrict__ Mt) {
  __shared__ __nv_bfloat16 t[64][66];
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = ty + 8 * i;
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(M + (r0 + row) * ld + c0 + 2 * tx);
    t[row][2 * tx] = v.x;
    t[row][2 * tx + 1] = v.y;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int col = ty + 8 * i;
    __nv_bfloat162 v;
    v.x = t[2 * tx][col];
    v.y = t[2 * tx + 1][col];
    *reinterpret_cast<__nv_bfloat162*>(Mt + (c0 + col) * r + r0 + 2 * tx) = v;
  }
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

  // split the long dimension of the sampled sketch into chunks of 128 columns, so that
  // (row blocks x chunks) fills the GPU even with l_k = 82 rows
  const int64_t split_len = 128;
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
  need += (size_t)kMaxW * kMaxW * 8 * 3 + small_solver_doubles(kMaxW) * 8 + 2048;  // G, T, Vr, solver scratch
  need += 64 * 4 * 2 + (2 + kMaxW) * 8 + 1024;                    // S, flags, factor stats
  need += jac_rot_entries(kJacMaxNE) * sizeof(double2) + 256;     // recorded Jacobi rotations
  need += (size_t)kMaxW * (4 + 8) + 1024;                          // Jacobi order, lambda^-1/2, info
  const int kpw = pad_width(std::max(w, k));
  const bool unsampled = lk >= r;   // the refresh's Bm^T = M^T Q then runs on M^T (tensor cores)
  need += (size_t)2 * kpw * std::max(r, c) * 2 + 256;             // hi/lo transposed operand
  // the largest split count of the projections below: M Omega and M V (widths w and k), and
  // M^T Q for the unsampled operand
  const int splits_est =
      std::max({normalize_splits(c, bf16_splits(ctx, r, c, 2 * pad_width(w))),
                normalize_splits(c, bf16_splits(ctx, r, c, 2 * pad_width(k))),
                unsampled ? normalize_splits(r, bf16_splits(ctx, c, r, 2 * pad_width(w))) : 1});
  const size_t tc_partial_bytes = (size_t)splits_est * std::max(r, c) * 2 * kpw * 4;
  need += tc_partial_bytes + 256;                                 // split partials
  if (unsampled) need += (size_t)r * c * 2 + 256;                 // M^T
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
  double* sscratch = static_cast<double*>(ws.take(small_solver_doubles(kMaxW) * 8));
  float* Sw = static_cast<float*>(ws.take(64 * 4));
  int* flags = static_cast<int*>(ws.take(64 * 4));
  unsigned long long* stats = static_cast<unsigned long long*>(ws.take((2 + kMaxW) * sizeof(unsigned long long)));
  double2* jrot = static_cast<double2*>(ws.take(jac_rot_entries(kJacMaxNE) * sizeof(double2)));
  int* jorder = static_cast<int*>(ws.take((size_t)kMaxW * 4));
  double* jinv = static_cast<double*>(ws.take((size_t)kMaxW * 8));
  int* jinfo = static_cast<int*>(ws.take(64));
  __nv_bfloat16* bt2 = static_cast<__nv_bfloat16*>(ws.take((size_t)2 * kpw * std::max(r, c) * 2));
  float* tc_partial = static_cast<float*>(ws.take(tc_partial_bytes));
  __nv_bfloat16* Mt = unsampled ? static_cast<__nv_bfloat16*>(ws.take((size_t)r * c * 2)) : nullptr;
  if (!tc_partial) return fail(ctx, METIS_ERR_WORKSPACE, "decompose workspace layout");

  cudaError_t e = cudaFuncSetAttribute(chol_inverse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)chol_smem_bytes(kSmallMaxN));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(jacobi_rounds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)jac_smem_bytes(kJacMaxNE));
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(small solver)");
  SmallOut so{T, Vr, Sw, flags, sscratch};
  JacOut jo{jrot, jinfo, jorder, jinv};
  // mode 0: CholQR factor T = R^+; modes 1 and 2: SVD through the eigenproblem of G
  auto solve = [&](int n, int mode) {
    if (mode == 0) {
      if (n <= kSmallMaxN) chol_inverse_kernel<<<1, kCholThreads, chol_smem_bytes(n), st>>>(G, n, so);
      else cholqr_solver_kernel<<<1, kSolverThreads, 0, st>>>(G, n, so);
    } else if (jac_ne(n) <= kJacMaxNE) {
      jacobi_rounds_kernel<<<1, kJacThreads, jac_smem_bytes(jac_ne(n)), st>>>(G, n, k, mode, jo, so, ctx->status,
                                                                          kJacobiMaxSweeps);
      count_launch();
      jacobi_replay_kernel<<<(n + kJacRowsPerCta - 1) / kJacRowsPerCta, 32 * kJacRowsPerCta, 0, st>>>(
          jrot, jinfo, n, k, mode, jorder, jinv, so);
    } else {
      eig_solver_kernel<<<1, kEigThreads, 0, st>>>(G, n, k, mode, so, ctx->status);
    }
    count_launch();
  };

  auto gram = [&](const float* A, int64_t n, int width) {
    const int64_t chunks = (n + kGramRows - 1) / kGramRows;
    const int64_t per_block = ((chunks + ctx->sm_count - 1) / ctx->sm_count) * kGramRows;
    const int nb = (int)((n + per_block - 1) / per_block);
    if (width <= 64) gram_partial_kernel<1><<<nb, 256, 0, st>>>(A, n, width, per_block, gpart, ctx->status);
    else gram_partial_kernel<4><<<nb, 256, 0, st>>>(A, n, width, per_block, gpart, ctx->status);
    count_launch();
    gram_reduce_kernel<<<(unsigned)((width * width + 7) / 8), 256, 0, st>>>(gpart, nb, width, G); count_launch();
  };
  // out (r x width) = M B on the tensor cores: B (c x width fp32) as a bf16 hi/lo pair
  // out (rows x width) = A B on the tensor cores: A bf16 (rows x K, leading dimension lda),
  // B fp32 (K x width) as a bf16 hi/lo pair, split-K partials summed in order
  auto project_on = [&](const __nv_bfloat16* A, int64_t lda, int64_t rows, int64_t K, const float* B, int width,
                        float* out) -> metis_status {
    const int kp = pad_width(width);
    split_hi_lo_t_kernel<<<(unsigned)((K + kSplitRows - 1) / kSplitRows), kSplitThreads, 0, st>>>(B, K, width, kp,
                                                                                              bt2);
    count_launch();
    const int splits = normalize_splits(K, bf16_splits(ctx, rows, K, 2 * kp));
    if (splits > kMaxProjSplits) return fail(ctx, METIS_ERR_ARG, "projection split count above the reduction's limit");
    if ((size_t)splits * rows * 2 * kp * 4 > tc_partial_bytes)
      return fail(ctx, METIS_ERR_WORKSPACE, "projection partials exceed workspace");
    metis_status st2 = launch_gemm_bf16(ctx, A, lda, rows, bt2, K, 2 * kp, K, tc_partial, 2 * kp, splits);
    if (st2 != METIS_OK) return st2;
    reduce_hi_lo_kernel<<<blocks_for(rows * width), 256, 0, st>>>(tc_partial, splits, rows, kp, width, out);
    count_launch();
    return METIS_OK;
  };
  // out (r x width) = M B
  auto project = [&](const float* B, int width, float* out) -> metis_status {
    return project_on(Mb, M->ld, r, c, B, width, out);
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
    solve(w, 0);
    times_small_kernel<<<blocks_for(lk * w), 256, 0, st>>>(Y, lk, w, T, w, Q); count_launch();
    // Bm^T = M_s^T Q ; R2 = chol(Bm Bm^T) ; SVD(R2^T) ; V = Bm^T R2^+ W'[:, :k]
    if (unsampled) {
      // all rows: Bm^T = M^T Q on the tensor cores, from one transposed copy of M
      dim3 tgrid((unsigned)(c / 64), (unsigned)(r / 64));
      transpose_bf16_kernel<<<tgrid, 256, 0, st>>>(Mb, M->ld, r, Mt); count_launch();
      if ((s = project_on(Mt, r, c, r, Q, w, Bt)) != METIS_OK) return s;
    } else {
      cols_times_matrix_kernel<<<blocks_for(c, 64), 256, 0, st>>>(Mb, M->ld, idx, lk, c, Q, w, Bt); count_launch();
    }
    gram(Bt, c, w);
    solve(w, 1);
    times_small_kernel<<<blocks_for(c * k), 256, 0, st>>>(Bt, c, w, T, k, f->V); count_launch();
  }
  // per step: P = M V ; R = chol(P^T P) ; SVD(R) ; U = P R^+ U_r ; V <- V V_r
  cudaEvent_t pev0 = nullptr, pev1 = nullptr;
  if (ctx->profiling) {
    cudaEventCreate(&pev0);
    cudaEventCreate(&pev1);
    cudaEventRecord(pev0, st);
  }
  if ((s = project(f->V, k, Y)) != METIS_OK) return s;
  if (ctx->profiling) {   // algorithmic bytes: one bf16 read of M
    cudaEventRecord(pev1, st);
    profile_record(ctx, kProfProjection, pev0, pev1, 2.0 * (double)r * (double)c);
  }
  gram(Y, r, k);
  so.S = f->S;
  solve(k, 2);
  // U = P T and V V_r, then the sign convention and the NVFP4 copies (blocks along the long
  // dimension, power-of-two tensor scale)
  FactorStats fs{stats, stats + 2};
  e = cudaMemsetAsync(stats, 0, (size_t)(2 + k) * sizeof(unsigned long long), st);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaMemsetAsync(factor stats)");
  e = cudaFuncSetAttribute(factor_products_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFpSmem);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(factor products)");
  factor_products_kernel<<<(unsigned)((r + kFpRows - 1) / kFpRows + (c + kFpRows - 1) / kFpRows), 256, kFpSmem,
                           st>>>(Y, r, T, f->V, c, Vr, k, Q, Bt, fs, ctx->status); count_launch();
  factor_finalize_kernel<<<(unsigned)((128 * (r / 16) + 128 * (c / 16) + 255) / 256), 256, 0, st>>>(
      Q, r, Bt, c, k, fs, p->rounding, p->seed, stream_tag(p->operand_id, kPurposeSR, kSrLeft),
      stream_tag(p->operand_id, kPurposeSR, kSrRight), step, f->U, f->V, f->Uq, f->Vq); count_launch();
  return check_cuda(ctx, cudaGetLastError(), "decompose");
}

// ---- self-test of the numeric-failure latch ----
namespace {
// G = the n x n matrix with 2 on the diagonal and 1 elsewhere (symmetric positive
// definite, far from diagonal)
__global__ void numeric_selftest_fill_kernel(double* G, int n) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n * n) G[e] = (e / n == e % n) ? 2.0 : 1.0;
}
}  // namespace

metis_status launch_numeric_selftest(metis_ctx* ctx) {
  constexpr int n = 8;
  const size_t need = (size_t)n * n * 8 + jac_rot_entries(n) * sizeof(double2) + (size_t)2 * n * kMaxW * 8 +
                      (size_t)kMaxW * (4 + 4 + 8 + 4) + 8 * 256;
  metis_status s = ensure_workspace(ctx, need);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  double* G = static_cast<double*>(ws.take((size_t)n * n * 8));
  double2* rot = static_cast<double2*>(ws.take(jac_rot_entries(n) * sizeof(double2)));
  double* T = static_cast<double*>(ws.take((size_t)n * kMaxW * 8));
  double* Vr = static_cast<double*>(ws.take((size_t)n * kMaxW * 8));
  float* S = static_cast<float*>(ws.take((size_t)kMaxW * 4));
  int* flags = static_cast<int*>(ws.take((size_t)kMaxW * 4));
  int* order = static_cast<int*>(ws.take((size_t)kMaxW * 4));
  double* inv = static_cast<double*>(ws.take((size_t)kMaxW * 8));
  int* info = static_cast<int*>(ws.take(64));
  if (!info) return fail(ctx, METIS_ERR_WORKSPACE, "numeric self-test workspace layout");
  cudaStream_t st = ctx->stream;
  numeric_selftest_fill_kernel<<<1, 64, 0, st>>>(G, n);
  count_launch();
  cudaError_t e = cudaFuncSetAttribute(jacobi_rounds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)jac_smem_bytes(kJacMaxNE));
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(numeric self-test)");
  SmallOut so{T, Vr, S, flags, nullptr};
  JacOut jo{rot, info, order, inv};
  // a sweep limit of zero: the solve stops before its first sweep, unconverged
  jacobi_rounds_kernel<<<1, kJacThreads, jac_smem_bytes(jac_ne(n)), st>>>(G, n, n, 2, jo, so, ctx->status, 0);
  count_launch();
  return check_cuda(ctx, cudaGetLastError(), "numeric self-test launch");
}

// ---- launchers shared with the LoRA-SVD calls (lora.cu) ----

cudaError_t launch_transpose_bf16(const void* M, int64_t ld, int64_t r, int64_t c, void* Mt, cudaStream_t st) {
  transpose_bf16_kernel<<<dim3((unsigned)(c / 64), (unsigned)(r / 64)), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(M), ld, r, static_cast<__nv_bfloat16*>(Mt));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_split_hi_lo_t(const float* F, int64_t n, int k, int kp, void* out, cudaStream_t st) {
  split_hi_lo_t_kernel<<<(unsigned)((n + kSplitRows - 1) / kSplitRows), kSplitThreads, 0, st>>>(
      F, n, k, kp, static_cast<__nv_bfloat16*>(out));
  count_launch();
  return cudaGetLastError();
}

size_t gram_scratch_doubles(metis_ctx* ctx, int w) { return (size_t)(ctx->sm_count + 1) * w * w; }

metis_status launch_gram(metis_ctx* ctx, const float* A, int64_t n, int w, double* scratch, double** G_out) {
  if (w < 1 || w > 64) return fail(ctx, METIS_ERR_SHAPE, "Gram width must be in [1, 64]");
  cudaStream_t st = ctx->stream;
  double* gpart = scratch;
  double* G = gpart + (size_t)ctx->sm_count * w * w;
  const int64_t chunks = (n + kGramRows - 1) / kGramRows;
  const int64_t per_block = ((chunks + ctx->sm_count - 1) / ctx->sm_count) * kGramRows;
  const int nb = (int)((n + per_block - 1) / per_block);
  gram_partial_kernel<1><<<nb, 256, 0, st>>>(A, n, w, per_block, gpart, ctx->status); count_launch();
  gram_reduce_kernel<<<(unsigned)((w * w + 7) / 8), 256, 0, st>>>(gpart, nb, w, G); count_launch();
  *G_out = G;
  return check_cuda(ctx, cudaGetLastError(), "Gram");
}

}  // namespace metis
