/*
 * libmetis -- the Metis spectral-domain W4A4G4 linear layer on NVIDIA B200.
 *
 * Method: "Metis: Training LLMs with FP4 Quantization" (ICLR 2026; papernotes.org
 * notes).  Every matrix M of a GeMM (weight W, activation X, output gradient D)
 * is split into a rank-k dominant part kept in high precision and a residual
 * quantized to NVFP4 (key design 1):
 *
 *     M = U_k S_k V_k^T + M_R
 *     Y = (Q(A_k) L_k Q(B_k^T) + Q(X_R)) (Q(U_k) S_k Q(V_k^T) + Q(W_R))
 *
 * with Q the NVFP4 block quantizer (E2M1 values, 16-element blocks, one E4M3
 * scale per block; background section) and the singular values kept in fp32.
 * The dominant subspace comes from l_k sampled rows and a Gaussian sketch of
 * width k + s (key design 2) and is reused across steps (key design 3).
 *
 * Conventions for every call:
 *   - All matrix pointers are DEVICE pointers owned by the caller; libmetis never
 *     allocates or frees them.  The context owns only its workspace and a device
 *     status word.
 *   - Calls are asynchronous on the context's stream.  The returned status covers
 *     host-side validation and launch only; numeric failures found on the device
 *     latch bits of the status word (METIS_DEV_*), read by
 *     metis_poll_device_status.  No kernel traps.
 *   - Shapes: every matrix dimension is a multiple of 128 (and, where it is a GeMM
 *     contraction length, of 256); 1 <= k <= 64; k + s <= 128; k + s <= l_k <= rows.
 *   - Alignment: pointers 16-byte aligned; bf16 leading dimensions a multiple of 8
 *     elements, fp32 ones a multiple of 4.
 *   - Device: sm_100 (B200) only; anything else returns METIS_ERR_ARCH.
 *   - On error nothing is launched and metis_last_error() describes the cause.
 */
#ifndef METIS_H
#define METIS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  METIS_OK = 0,
  METIS_ERR_ARG = 1,        /* null pointer, bad enum or inconsistent descriptor */
  METIS_ERR_SHAPE = 2,      /* a dimension outside the limits above */
  METIS_ERR_ALIGN = 3,      /* pointer or leading-dimension alignment */
  METIS_ERR_ARCH = 4,       /* device is not sm_100 */
  METIS_ERR_CUDA = 5,       /* a CUDA runtime or driver call failed */
  METIS_ERR_WORKSPACE = 6   /* the context could not grow its workspace */
} metis_status;

/* Bits of the device status word (latched; cleared by metis_poll_device_status). */
#define METIS_DEV_NUMERIC   1u  /* a small dense factorization did not converge */
#define METIS_DEV_NONFINITE 2u  /* NaN or Inf met in a quantizer or decomposition input */
#define METIS_DEV_TIMEOUT   4u  /* a bounded wait inside a kernel ran out; its work was skipped */

typedef struct metis_ctx metis_ctx;

/* Creates a context on `device` issuing work on `stream` (a cudaStream_t, may be 0).
 * Fails with METIS_ERR_ARCH unless the device is sm_100. */
metis_status metis_create(int device, void* stream, metis_ctx** out);
/* Frees the context's workspace and status word (synchronizes its stream). */
void metis_destroy(metis_ctx* ctx);
metis_status metis_set_stream(metis_ctx* ctx, void* stream);
/* Sizes this context's later launches for n SMs instead of the device's count: the
 * persistent kernels (fused GeMM, residual quantizer, thin and projection GeMMs) launch
 * at most n CTAs (pairs: n / 2) and the split-K counts are chosen for n, so work the
 * caller runs on other streams at the same time keeps the remaining SMs (the counterpart
 * of a library's SM-count target). n = 0 restores the device's count; otherwise
 * 2 <= n <= the device's SM count, else METIS_ERR_ARG. Outputs of the quantizers and of
 * the fused GeMM do not depend on n; the fp32 sums of split-K products (projection,
 * Gram, fold preparation) may differ in their last bits, as their split count follows n.
 * Applies to calls issued after it; not thread-safe against calls in flight on ctx. */
metis_status metis_set_sm_count_target(metis_ctx* ctx, int n);
const char* metis_status_str(metis_status s);
/* Message of the last failed call on this context; owned by the context. */
const char* metis_last_error(const metis_ctx* ctx);
/* Synchronizes the stream, returns the latched METIS_DEV_* bits, clears them if `clear`. */
metis_status metis_poll_device_status(metis_ctx* ctx, uint32_t* bits, int clear);

/* Dense bf16 device matrix, row-major with leading dimension `ld` (elements). */
typedef struct {
  const void* data;
  int64_t rows, cols, ld;
} metis_matrix;

/*
 * NVFP4 tensor in one orientation: logically outer x inner with 16-element blocks
 * along inner (inner is the contraction dimension of the GeMM that reads it).
 *   codes  : outer x inner/2 bytes, row-major; element 2t of a row sits in the low
 *            nibble of byte t, element 2t+1 in the high nibble; code bit 3 = sign,
 *            bits 0-2 index the E2M1 magnitudes {0,0.5,1,1.5,2,3,4,6}.
 *   scales : E4M3 (OCP fn) block scales in 512-byte tiles, one tile per 128 rows x
 *            64 inner elements; tile (ob, kb) starts at byte (ob*(inner/64)+kb)*512
 *            and holds the scale of row o, block b at offset
 *            (o%32)*16 + ((o%128)/32)*4 + (b%4)  -- the layout the tcgen05
 *            block-scaled MMA reads from tensor memory.
 *   tensor_scale : device pointer to one fp32 decode-side tensor scale g (a power
 *            of two).  Decoded value = e2m1(code) * e4m3(scale) * g.
 */
typedef struct {
  uint8_t* codes;
  uint8_t* scales;
  float* tensor_scale;
  int64_t outer, inner;
} metis_nvfp4;

/* Bytes needed for the codes / scales of an outer x inner NVFP4 tensor. */
int64_t metis_nvfp4_codes_bytes(int64_t outer, int64_t inner);
int64_t metis_nvfp4_scales_bytes(int64_t outer, int64_t inner);

/*
 * Low-rank factors of one operand M (rows x cols):  U S V^T  (key design 1).
 *   V  : cols x k fp32 row-major -- the reused subspace basis (key design 3).  Input
 *        to every step, rotated in place within its span; overwritten on refresh.
 *   U  : rows x k fp32 (output of every step), S : k fp32 descending (output).
 *   Uq, Vq : NVFP4 of U^T and V^T (outer = 128, inner = rows / cols); rows >= k are
 *        zero.  Blocks run along the long dimension; tensor scale is the smallest
 *        power of two g with max|F| <= 6*448*g (set on the device).
 *   sampled_rows (l_k int32) and omega (cols x (k+s) fp32): optional (nullable)
 *        copies of the last refresh's row sample and Gaussian test matrix.
 */
typedef struct {
  int64_t rows, cols;
  int32_t k;
  float* V;
  float* U;
  float* S;
  metis_nvfp4 Uq;
  metis_nvfp4 Vq;
  int32_t* sampled_rows;
  float* omega;
} metis_factors;

typedef struct {
  int32_t k;             /* rank (training strategy: 1.5% of the hidden size) */
  int32_t s;             /* sketch oversampling; sketch width k + s */
  int32_t l_k;           /* sampled rows (key design 2); l_k == rows disables sampling */
  uint64_t seed;         /* Philox4x32-10 key */
  uint32_t operand_id;   /* separates the random streams of X, W, D */
  int32_t rounding;      /* factor quantization: 0 round-to-nearest, 1 stochastic */
} metis_decomp_params;

/*
 * Randomized decomposition of M (key designs 2 and 3).
 * refresh != 0: sample l_k rows (Philox), draw Omega ~ N(0,1) (Philox + Box-Muller),
 *   sketch Y = M_s Omega, CholQR(Y) = Q R, Bm = Q^T M_s, CholQR(Bm^T) = Q2 R2,
 *   one-sided Jacobi SVD of R2^T, V = Q2 W'[:, :k].
 * Every call: P = M V, then the k x k symmetric eigenproblem of the Gram matrix
 *   G = P^T P = V_r diag(S_r^2) V_r^T (two-sided Jacobi in fp64; an eigenvalue at or
 *   below 1e-12 * lambda_max counts as zero and gives a zero column), U = P V_r
 *   diag(1 / S_r), S = S_r, V <- V V_r (sign-fixed), then Uq and Vq.  This equals the
 *   route CholQR(P) = Q_P R_P, SVD R_P = U_r S_r V_r^T, U = Q_P U_r of the method's
 *   statement (same U, S, V up to rounding and signs).
 * `step` enters the Philox counters (row sample, Omega, stochastic rounding).
 * Errors: ERR_SHAPE for k/s/l_k outside the limits; device: METIS_DEV_NONFINITE,
 * METIS_DEV_NUMERIC.
 */
metis_status metis_decompose(metis_ctx* ctx, const metis_matrix* M, const metis_decomp_params* p,
                             int refresh, uint32_t step, metis_factors* f);

typedef struct {
  int32_t rounding;      /* 0 round-to-nearest-even, 1 stochastic (training strategy) */
  uint64_t seed;
  uint32_t operand_id;
  uint32_t step;
  float tensor_scale;    /* decode-side tensor scale g (power of two, > 0), or 0: chosen from the
                            data as the smallest power of two with 2 * amax <= 6 * 448 * g, amax =
                            max |x| over the finite entries of the input (1 for an all-zero input,
                            exponent kept in [-126, 127]); costs one extra read of the input.  The
                            chosen g is written to the outputs' tensor_scale words. */
} metis_quant_params;

/*
 * Residual quantization (key design 1):  M_R = M - U diag(S) V^T  (factors f, fp32,
 * unquantized; f == NULL or f->k == 0 quantizes M itself -- plain NVFP4), then NVFP4
 * in one or both orientations:
 *   rowwise (nullable): outer = rows, inner = cols  (blocks along columns)
 *   colwise (nullable): outer = cols, inner = rows  (blocks along rows; M_R^T)
 * Stochastic rounding uses the Philox SR stream (operand_id, sub 0 row-wise / 1
 * column-wise, step).  With both orientations the pass runs fused (one read of M) and
 * needs rows * cols <= 2^36, else ERR_SHAPE.  Device: METIS_DEV_NONFINITE on NaN/Inf input.
 */
metis_status metis_residual_quantize_nvfp4(metis_ctx* ctx, const metis_matrix* M,
                                           const metis_factors* f, const metis_quant_params* q,
                                           metis_nvfp4* rowwise, metis_nvfp4* colwise);

/*
 * Parity surface of the residual quantization (key design 1): the same pass as
 * metis_residual_quantize_nvfp4 with both orientations, which also writes the fp32
 * residual that its quantizer rounded to `residual` (rows x cols, leading dimension ldr,
 * caller-owned device memory, 16-byte aligned, ldr % 4 == 0).  With k > 0 the pass
 * rebuilds U diag(S) V^T on the tensor cores from fp16 hi/lo splits of power-of-two
 * scaled 128-row blocks of U diag(S) and V (hi*hi + hi*lo + lo*hi, fp32 accumulation),
 * so this residual differs from M - U diag(S) V^T by about 2^-21 of the largest
 * reconstruction term; its NVFP4 codes and scales are exactly the block rule applied to
 * it.  Errors as metis_residual_quantize_nvfp4; ERR_ARG without both outputs and the
 * residual; ERR_ALIGN on the residual buffer.
 */
metis_status metis_residual_quantize_nvfp4_dump(metis_ctx* ctx, const metis_matrix* M,
                                                const metis_factors* f, const metis_quant_params* q,
                                                metis_nvfp4* rowwise, metis_nvfp4* colwise,
                                                float* residual, int64_t ldr);

/*
 * NVFP4 quantization of an fp32 device matrix R (rows x cols, leading dimension ld):
 * the quantizer alone, bit-exact with the block rule (background section; training
 * strategy for stochastic rounding).  Same outputs as above.
 */
metis_status metis_quantize_nvfp4_f32(metis_ctx* ctx, const float* R, int64_t rows, int64_t cols,
                                      int64_t ld, const metis_quant_params* q,
                                      metis_nvfp4* rowwise, metis_nvfp4* colwise);

/*
 * Decode of one NVFP4 tensor (background section: the value of an element is its E2M1
 * code times its block's E4M3 scale, times the decode tensor scale g):
 *   out[o * ld + i] = e2m1(code(o, i)) * e4m3(scale(o, i / 16)) * g
 * for the outer x inner tensor t; out is caller-owned fp32 device memory (16-byte
 * aligned, ld >= inner, ld % 4 == 0).  Exact: every product is an fp32 number.
 * Errors: ERR_SHAPE unless inner % 64 == 0; ERR_ALIGN on the output.
 */
metis_status metis_dequantize_nvfp4(metis_ctx* ctx, const metis_nvfp4* t, float* out, int64_t ld);

/*
 * Allocation-free residual quantization (no counterpart in the paper).
 * Same computation and results as metis_residual_quantize_nvfp4 with both
 * orientations, for callers that may not allocate device memory while they run:
 * a step being captured into a CUDA graph cannot call cudaMalloc, and a
 * framework that manages device memory through its own caching allocator must
 * not have a library allocate behind it.  This call allocates nothing: its
 * scratch (the fp16 hi/lo tiles of U diag(S) and V that the tensor cores read, and
 * their block factors) is a fixed 6 MiB device array inside libmetis, present on every
 * GPU that loads the library until the process exits.  The caller still provides every input and output.
 *   - rows + cols must not exceed 24576 (k <= 64); larger shapes return
 *     METIS_ERR_SHAPE with a message.  rowwise and colwise are both required.
 *   - The first call on a device looks up the array's device address (once per
 *     device, cached for the process).
 *   - All calls share the one array and it keeps the last call's contents (every
 *     call overwrites the part it reads first).  Calls whose GPU work overlaps --
 *     e.g. issued on two streams without ordering -- race on it.
 */
metis_status metis_residual_quantize_nvfp4_noalloc(metis_ctx* ctx, const metis_matrix* M,
                                                   const metis_factors* f, const metis_quant_params* q,
                                                   metis_nvfp4* rowwise, metis_nvfp4* colwise);

/* Output element types. */
#define METIS_OUT_F32  0
#define METIS_OUT_BF16 1

/*
 * Block-scaled FP4 GeMM with an optional bf16 rank-fold, the kernel behind the
 * layer calls:
 *   C[i][j] = alpha * col_scale[j] * ( sum_k A(i,k) B(j,k)  +  sum_t Fa[i][t] Fb[j][t] )
 * A: outer = p (rows of C); B: outer >= q (q = n_cols, the columns of C);
 * A.inner == B.inner = K, a multiple of 256.
 * A and B codes are decoded WITHOUT their tensor scales; alpha = gA * gB is read
 * from the devices' tensor_scale words.  Fa (p x fold_k) and Fb (q x fold_k) are
 * bf16 row-major device matrices (both NULL with fold_k == 0); fold_k is a
 * multiple of 64.  col_scale (q fp32) may be NULL (all ones).  C has leading
 * dimension ldc and type c_dtype (METIS_OUT_*).
 * q must be a multiple of 256, or one of 16, 32, 64 (thin GeMM; B.outer = 128 with
 * rows >= q zero).  col_scale, when given, holds q values.
 */
metis_status metis_gemm_nvfp4(metis_ctx* ctx, const metis_nvfp4* A, const metis_nvfp4* B, int64_t n_cols,
                              const void* Fa, const void* Fb, int32_t fold_k,
                              const float* col_scale, void* C, int64_t ldc, int32_t c_dtype);

/* One operand of the layer: residual in both orientations plus its factors
 * (f may be NULL or have k == 0 for plain NVFP4). */
typedef struct {
  const metis_nvfp4* rowwise;
  const metis_nvfp4* colwise;
  const metis_factors* f;
} metis_operand;

/*
 * Forward GeMM (key design 1 equation):  Y = X_hat W_hat  (l x n)
 *   X_hat = Q(A) L Q(B)^T + Q(X_R)_rowwise,   W_hat = Q(U) S Q(V)^T + Q(W_R)_colwise.
 * Evaluated as one FP4 GeMM Q(X_R) Q(W_R) plus the rank-fold of the low-rank terms
 * into the same accumulator.  Y has leading dimension ldy and type y_dtype.
 */
metis_status metis_linear_fwd(metis_ctx* ctx, const metis_operand* X, const metis_operand* W,
                              void* Y, int64_t ldy, int32_t y_dtype);

/*
 * Backward GeMMs (framework section: the split is embedded in every forward and
 * backward GeMM):  dX = D_hat W_hat^T  (l x m, type dx_dtype),  dW = X_hat^T D_hat
 * (m x n, fp32).  D uses its row-wise residual for dX and column-wise for dW; W its
 * row-wise residual; X its column-wise residual.
 */
metis_status metis_linear_bwd(metis_ctx* ctx, const metis_operand* X, const metis_operand* W,
                              const metis_operand* D, void* dX, int64_t lddx, int32_t dx_dtype,
                              float* dW, int64_t lddw);

/*
 * LoRA-SVD linear projection ("Full-Stack FP4", gist.science technical summary, section
 * 2.1): the weight is W = W_res + beta L2 L1 with the compact principal subspace L2 L1
 * (L2: m x k, L1: k x n, fp32 row-major masters, used in bf16 on the tensor cores) and
 * the residual W_res in NVFP4.  k in [1, 64].
 *
 * metis_lora_linear: one fused FP4 GeMM with the branch in its bf16 rank fold
 *   which = 0 (forward):        C = Q(A) Q(B)^T + beta (M bf16(L2)) bf16(L1)
 *       A = Q(X) row-wise (l x m), B = Q(W_res) column-wise (outer n, inner m), M = X.
 *   which = 1 (input gradient): C = Q(A) Q(B)^T + beta (M bf16(L1)^T) bf16(L2)^T
 *       A = Q(D) row-wise (l x n), B = Q(W_res) row-wise (outer m, inner n), M = D.
 *   Q(A) Q(B)^T is decoded with the tensor scales, as in metis_gemm_nvfp4.  T (nullable,
 *   l x k fp32): receives M bf16(L2) (which 0) or M bf16(L1)^T (which 1), the input of
 *   metis_lora_branch_grad.  B.outer (the columns of C) must be a multiple of 256; M is
 *   A.outer x A.inner bf16.  C: leading dimension ldc, type c_dtype.
 * metis_lora_branch_grad: G = beta M^T T (c x k fp32; transpose_out != 0 writes G^T,
 *   k x c) for M (p x c bf16) and T (p x k fp32), on the bf16 tensor cores (T as a bf16
 *   hi/lo pair).  With M = X and T from which = 1 this is dL/dL2 = beta X^T D L1^T; with
 *   M = D, T from which = 0 and transpose_out it is dL/dL1 = beta (X L2)^T D.
 * metis_lora_constrain: the Cholesky-QR constraint, in place: L2 = Q R (CholQR in fp64,
 *   dependent columns dropped), L2 <- Q, L1 <- R L1; the product L2 L1 is unchanged up
 *   to rounding and L2 has orthonormal columns.
 * metis_lora_realign: randomized-SVD realignment, in place.  W_eff = W_res + beta L2 L1
 *   (fp32, leading dimension ldw); bf16(W_eff) is written to W_bf16 (m x n, caller
 *   scratch) and decomposed by metis_decompose with refresh (params p, k = p->k, the
 *   caller's factors f of shape m x n as buffers) into U S V^T; then L2 <- U,
 *   L1 <- diag(S / beta) V^T and W_res <- W_eff - beta L2 L1 (fp32), so W_res + beta L2 L1
 *   equals W_eff up to fp32 rounding.  beta must be nonzero.
 * Errors: ERR_ARG (null, bad which, non-finite beta), ERR_SHAPE, ERR_ALIGN (16-byte
 * aligned buffers).  Device: as metis_decompose for the realignment.
 */
metis_status metis_lora_linear(metis_ctx* ctx, int32_t which, const metis_nvfp4* A, const metis_nvfp4* B,
                               const metis_matrix* M, const float* L2, const float* L1, int32_t k, float beta,
                               float* T, void* C, int64_t ldc, int32_t c_dtype);
metis_status metis_lora_branch_grad(metis_ctx* ctx, const metis_matrix* M, const float* T, int32_t k, float beta,
                                    int32_t transpose_out, float* G);
metis_status metis_lora_constrain(metis_ctx* ctx, float* L2, int64_t m, float* L1, int64_t n, int32_t k);
metis_status metis_lora_realign(metis_ctx* ctx, float* W_res, int64_t m, int64_t n, int64_t ldw, float* L2,
                                float* L1, int32_t k, float beta, const metis_decomp_params* p, uint32_t step,
                                metis_factors* f, void* W_bf16);

/*
 * Self-test of failure detection (no counterpart in the notes).  Every wait of the
 * tensor-core kernels is bounded: on expiry the kernel sets METIS_DEV_TIMEOUT in the
 * context's status word and returns normally.  This launches one CTA that waits on a
 * barrier nothing arrives at, with a limit of `limit_cycles` SM clock cycles
 * (1 .. 2e8, about 0.1 s at most), so the caller can check that the timeout is reported
 * by metis_poll_device_status and that the context stays usable.
 * Errors: ERR_ARG for a limit outside the range.
 */
metis_status metis_selftest_wait_timeout(metis_ctx* ctx, int64_t limit_cycles);

/*
 * Self-test of the numeric-failure latch (no counterpart in the notes).  The small
 * eigensolver latches METIS_DEV_NUMERIC when a solve reaches its sweep limit unconverged.
 * This runs it, on the context's stream, on a fixed 8 x 8 symmetric matrix (2 on the
 * diagonal, 1 elsewhere) with the limit set to zero sweeps, so the solve stops at once,
 * raises the bit and returns normally; the caller checks metis_poll_device_status and
 * that the context stays usable.  Uses the context's workspace (grown if needed).
 * Errors: ERR_WORKSPACE if the workspace cannot grow.
 */
metis_status metis_selftest_numeric(metis_ctx* ctx);

/*
 * NVFP4 tensor-core throughput microbenchmark (no counterpart in the notes; the measured
 * ceiling for the fused GeMM).  Launches, on the context's stream, one cluster of two
 * CTAs per SM pair; each pair issues `iters` stages of four block-scaled MMAs
 * (tcgen05 kind::mxf4nvf4, block16, M = 256, N = 256, K = 64) on operands resident in
 * shared and tensor memory, with no memory traffic.  *flops receives the useful flops
 * of the launch (2 * 256 * 256 * 256 * iters per pair); the caller times the launch.
 * Errors: ERR_ARG for iters < 1 or more than 2^20 (keeps one launch well under a second).
 */
metis_status metis_nvfp4_mma_peak(metis_ctx* ctx, int64_t iters, double* flops);

/*
 * Instrumentation (the notes have no counterpart; used by the benchmark).
 * metis_kernel_launches: number of kernels libmetis has launched in this process.
 * metis_profile_enable: when on, the launches of three kernels are bracketed by CUDA
 *   events on the context's stream: every main GeMM (the fused FP4 + fold kernel of
 *   the layer calls and metis_gemm_nvfp4 with n_cols >= 256; METIS_PROF_GEMM), every
 *   two-orientation residual quantization pass (METIS_PROF_RESQUANT) and every per-step
 *   projection P = M V of metis_decompose (METIS_PROF_PROJECTION).
 * metis_profile_read_kind: synchronizes the stream and returns, for one kind, the summed
 *   event time (ms), the number of timed launches and their algorithmic work -- flops
 *   2*p*q*K for the GeMM, bytes for the two HBM-bound kernels (3.125 per element of M
 *   for the quantizer: 2 read, 2 x (1/2 + 1/16) written; 2 per element of M read for the
 *   projection) -- then resets that kind's record.  metis_profile_read is the GeMM kind.
 */
#define METIS_PROF_GEMM       0
#define METIS_PROF_RESQUANT   1
#define METIS_PROF_PROJECTION 2
uint64_t metis_kernel_launches(void);
metis_status metis_profile_enable(metis_ctx* ctx, int on);
metis_status metis_profile_read(metis_ctx* ctx, double* ms, int64_t* launches, double* flops);
metis_status metis_profile_read_kind(metis_ctx* ctx, int32_t kind, double* ms, int64_t* launches,
                                     double* work);

#ifdef __cplusplus
}
#endif

#endif /* METIS_H */
