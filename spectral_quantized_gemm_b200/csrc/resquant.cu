// Fused residual + NVFP4 quantization in both orientations (one read of M).
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
// key design 1: M = U S V^T + M_R with the residual M_R quantized to NVFP4
// (background section: E2M1, 16-element blocks, E4M3 block scale; training
// strategy: stochastic rounding).  Every residual is quantized twice, with
// blocks along each GeMM contraction dimension that reads it.
//
// Per 128 x 128 tile of M (persistent CTAs, contiguous row-block-major ranges):
//   warp 0      TMA: the U*S rows of the row block (kept while the block lasts),
//               then per tile the V rows and the two 64-column boxes of M (3 stages)
//   warp 1      tensor-memory owner; one thread issues tcgen05.mma kind::tf32 for the
//               reconstruction (U S) V^T and for its transpose V (U S)^T, each into a
//               double-buffered fp32 accumulator (the same operands, swapped)
//   warps 2..17 a warp per 32 x 32 sub-tile: row-wise quantization of M - (U S) V^T from
//               its rows (reconstruction rows from tensor memory, M rows from shared
//               memory), then column-wise quantization of the same sub-tile from the
//               transposed reconstruction and M's columns; codes and tiled scales go
//               straight to HBM.  The warps never wait for one another.
// All mbarrier waits are bounded (METIS_DEV_TIMEOUT on expiry).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace metis {
namespace {

constexpr int kRqEpiWarps = 16;                 // 4 per tensor-memory lane quarter
constexpr int kRqEpiThreads = kRqEpiWarps * 32;
constexpr int kRqThreads = 64 + kRqEpiThreads;

template <int KK>
struct RqCfg {
  static constexpr int A_BYTES = 128 * KK * 4;   // KK/32 swizzle atoms of 128 rows x 128 B
  static constexpr int V_BYTES = 128 * KK * 4;
  static constexpr int M_BYTES = 128 * 128 * 2;  // two 64-column boxes of 16 KB
  static constexpr int STAGE_BYTES = V_BYTES + M_BYTES;
  static constexpr int STAGES = 3;
  static constexpr size_t SMEM = (size_t)A_BYTES + STAGES * STAGE_BYTES + 1024 + 256 + 512;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct RqParams {
  int64_t rows, cols;
  int n_cb, n_units;
  float g;
  int rounding;
  uint64_t seed;
  uint32_t tag_row, tag_col, step;
  uint8_t* row_codes;
  uint8_t* row_scales;
  uint8_t* col_codes;
  uint8_t* col_scales;
  float* row_g;
  float* col_g;
  const uint32_t* amax_bits;   // non-null: g chosen from the data (auto_tensor_scale)
  uint32_t* status;
};

__host__ __device__ __forceinline__ uint32_t idesc_tf32(uint32_t n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The block rule of block_scale() with two exact shortcuts for this kernel:
//  * target = RN(amax / (6 g)).  For g = 1 it is formed as q0 = RN(amax * RN(1/6)) corrected
//    by one fused multiply-add, q0 + RN(amax - 6 q0) * RN(1/6); checked exhaustively on the
//    CPU to equal the IEEE quotient for every finite amax >= 2^-125, and below that both
//    round to E4M3 code 0.  Other g use the IEEE division.
//  * rcp = RN(1 / (s g)) depends only on the scale code: a per-CTA table of 128 entries
//    built with the same operations.
__device__ __forceinline__ BlockScale block_scale_fast(float amax, float g, const float* rcp_table) {
  float target;
  if (g == 1.0f) {
    const float r6 = 1.0f / 6.0f;
    const float q0 = __fmul_rn(amax, r6);
    target = __fmaf_rn(__fmaf_rn(-6.0f, q0, amax), r6, q0);
  } else {
    target = __fdiv_rn(amax, __fmul_rn(6.0f, g));
  }
  uint32_t code = e4m3_code_rn(target);
  if (amax > 0.0f && code == 0) code = 1;  // smallest E4M3 value 2^-9
  BlockScale bs;
  bs.code = code;
  bs.rcp = rcp_table[code & 127u];
  return bs;
}

// One 16-element block: scale code and packed codes (RN or SR with the Philox
// stream of element index e0 .. e0 + 15 in the orientation's blocked order).  amax is
// the block's largest |v| (computed by the caller).
__device__ __forceinline__ uint2 quantize16(const float (&v)[16], float amax, float g, const float* rcp_table,
                                            int rounding, uint64_t seed, uint32_t tag, uint32_t step, uint64_t e0,
                                            uint32_t& scale_code) {
  const BlockScale bs = block_scale_fast(amax, g, rcp_table);
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __fmul_rn(v[i], bs.rcp);
  uint2 packed = encode_block16(x, rounding, seed, tag, step, e0);
  if (bs.code == 0) packed = make_uint2(0, 0);
  scale_code = bs.code;
  return packed;
}

template <int KK>
__global__ void __launch_bounds__(kRqThreads, 1)
    resquant_kernel(const __grid_constant__ CUtensorMap mapM, const __grid_constant__ CUtensorMap mapUS,
                    const __grid_constant__ CUtensorMap mapV, const RqParams p) {
  using C = RqCfg<KK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sStage = sA + C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + C::STAGES * C::STAGE_BYTES);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* full = bars + 2;                 // [STAGES]
  uint64_t* empty = full + C::STAGES;        // [STAGES]
  uint64_t* acc_full = empty + C::STAGES;    // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rcp_table = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);   // 128 entries

  const float g = p.amax_bits ? auto_tensor_scale(*p.amax_bits) : p.g;
  for (int c = threadIdx.x; c < 128; c += blockDim.x)
    rcp_table[c] = c ? __frcp_rn(__fmul_rn(e4m3_value((uint32_t)c), g)) : 0.0f;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int per = (p.n_units + gridDim.x - 1) / gridDim.x;
  const int u_begin = blockIdx.x * per;
  const int u_end = min(p.n_units, u_begin + per);

  if (threadIdx.x == 0) {
    tc::mbar_init(a_full, 1);
    tc::mbar_init(a_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1 + kRqEpiThreads / 32);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], kRqEpiThreads / 32);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    if (blockIdx.x == 0) {
      *p.row_g = g;
      *p.col_g = g;
    }
  }
  if (warp == 1) {   // columns 0-255: reconstruction, 256-511: its transpose (two buffers each)
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail_wait = [&]() {
    *abort_flag = 1;
    raise_status(p.status, METIS_DEV_TIMEOUT);
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, a_phase = 0;
      int cur_rb = -1;
      for (int u = u_begin; u < u_end && !*abort_flag; ++u) {
        const int rb = u / p.n_cb, cb = u % p.n_cb;
        if (rb != cur_rb) {
          if (!tc::mbar_wait(a_empty, a_phase ^ 1u, abort_flag)) { fail_wait(); break; }
          tc::mbar_expect_tx(a_full, C::A_BYTES);
#pragma unroll
          for (int ch = 0; ch < KK / 32; ++ch) tc::tma_load_2d(sA + ch * 16384, &mapUS, a_full, ch * 32, rb * 128);
          a_phase ^= 1u;
          cur_rb = rb;
        }
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { fail_wait(); break; }
        uint8_t* sV = sStage + stage * C::STAGE_BYTES;
        uint8_t* sM = sV + C::V_BYTES;
        tc::mbar_expect_tx(&full[stage], C::STAGE_BYTES);
#pragma unroll
        for (int ch = 0; ch < KK / 32; ++ch) tc::tma_load_2d(sV + ch * 16384, &mapV, &full[stage], ch * 32, cb * 128);
        tc::tma_load_2d(sM, &mapM, &full[stage], cb * 128, rb * 128);
        tc::tma_load_2d(sM + 16384, &mapM, &full[stage], cb * 128 + 64, rb * 128);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, a_phase = 0;
      int cur_rb = -1;
      int it = 0;
      const uint32_t idesc = idesc_tf32(128);
      for (int u = u_begin; u < u_end && !*abort_flag; ++u, ++it) {
        const int rb = u / p.n_cb;
        if (rb != cur_rb) {
          if (cur_rb >= 0) tc::tc_commit(a_empty);  // the old U*S rows are no longer read
          if (!tc::mbar_wait(a_full, a_phase, abort_flag)) { fail_wait(); break; }
          a_phase ^= 1u;
          cur_rb = rb;
        }
        const int b = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!tc::mbar_wait(&full[stage], phase, abort_flag)) { fail_wait(); break; }
        if (!tc::mbar_wait(&acc_empty[b], (use & 1u) ^ 1u, abort_flag)) { fail_wait(); break; }
        tc::tc_fence_after();
        const uint8_t* sV = sStage + stage * C::STAGE_BYTES;
#pragma unroll
        for (int ch = 0; ch < KK / 32; ++ch) {
          const uint64_t ad = tc::sdesc_sw128(tc::smem_addr(sA + ch * 16384));
          const uint64_t bd = tc::sdesc_sw128(tc::smem_addr(sV + ch * 16384));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mma_tf32(tmem + b * 128, ad + 2 * j, bd + 2 * j, idesc, (ch | j) ? 1u : 0u);          // rows of the tile
            mma_tf32(tmem + 256 + b * 128, bd + 2 * j, ad + 2 * j, idesc, (ch | j) ? 1u : 0u);    // its columns
          }
        }
        tc::tc_commit(&empty[stage]);
        tc::tc_commit(&acc_full[b]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      tc::tc_commit(drain);
      tc::mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;            // tensor-memory lane quarter
    const int h = (warp - 2) >> 2;     // 32-column quarter (row pass) = 32-row quarter (column pass)
    const int r = q * 32 + lane;       // tile row of this thread in the row pass
    const int j = q * 32 + lane;       // tile column of this thread in the column pass
    // M(i, j) of the column pass sits in box j >> 6 at row i, 16-byte chunk
    // ((j & 63) >> 3) ^ (i & 7), element j & 7: the 8 chunk positions, by i & 7
    const int jc = (j & 63) >> 3;
    uint32_t col_off[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) col_off[t] = (uint32_t)((j >> 6) * 16384 + (((jc ^ t) << 4) | ((j & 7) << 1)));
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int u = u_begin; u < u_end; ++u, ++it) {
      const int rb = u / p.n_cb, cb = u % p.n_cb;
      const int b = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      bool ok = tc::mbar_wait(&acc_full[b], use & 1u, abort_flag);
      ok = ok && tc::mbar_wait(&full[stage], phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail_wait();
        break;
      }
      tc::tc_fence_after();
      const uint8_t* sM = sStage + stage * C::STAGE_BYTES + C::V_BYTES;
      // ---- row-wise quantization (blocks along columns): row r, columns h*32 .. + 31
      {
        float v[32];
        tc::tmem_load_32cols(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 128 + h * 32), v);
        tc::tmem_load_wait();
        // residual = M - reconstruction (M from the 128B-swizzled 64-column box holding
        // this quarter: chunks (h & 1) * 4 .. + 3 of box h >> 1)
        const uint8_t* sMb = sM + (h >> 1) * 16384;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = (h & 1) * 4 + cc;
          const uint4 raw = *reinterpret_cast<const uint4*>(sMb + r * 128 + ((c ^ (r & 7)) << 4));
          const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(pr[i]);
            v[cc * 8 + 2 * i] = f.x - v[cc * 8 + 2 * i];
            v[cc * 8 + 2 * i + 1] = f.y - v[cc * 8 + 2 * i + 1];
          }
        }
        const int64_t grow = (int64_t)rb * 128 + r;
        const int64_t gcol = (int64_t)cb * 128 + h * 32;
        uint32_t sc = 0;
        uint4 out;
        uint32_t* o = reinterpret_cast<uint32_t*>(&out);
        bool finite = true;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float x[16];
          // block maximum of |x|: fmaxf keeps an Inf but drops a NaN, which a sum of the
          // block's magnitudes then shows (the sum is NaN exactly when an element is)
          float amax = 0.0f, sum = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            x[i] = v[blk * 16 + i];
            amax = fmaxf(amax, fabsf(x[i]));
            sum += fabsf(x[i]);
          }
          finite &= (amax <= 3.402823466e38f) && (sum == sum);
          uint32_t code;
          const uint2 pk = quantize16(x, amax, g, rcp_table, p.rounding, p.seed, p.tag_row,
                                      p.step, (uint64_t)grow * (uint64_t)p.cols + (uint64_t)(gcol + blk * 16), code);
          sc |= code << (8 * blk);
          o[2 * blk] = pk.x;
          o[2 * blk + 1] = pk.y;
        }
        if (!finite) raise_status(p.status, METIS_DEV_NONFINITE);
        *reinterpret_cast<uint4*>(p.row_codes + grow * (p.cols / 2) + gcol / 2) = out;
        *reinterpret_cast<uint16_t*>(p.row_scales + scale_offset(grow, gcol / 16, p.cols / 64)) = (uint16_t)sc;
      }
      // ---- column-wise quantization (blocks along rows): column j, rows h*32 .. + 31,
      // from the transposed reconstruction (tensor-memory lane j) and M's column j
      {
        const uint8_t* cbase[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) cbase[t] = sM + h * 32 * 128 + col_off[t];
        float w[32];
        tc::tmem_load_32cols(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(256 + b * 128 + h * 32), w);
        tc::tmem_load_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&acc_empty[b]);   // both reconstructions of this tile are read
        const int64_t gcolj = (int64_t)cb * 128 + j;
        const int64_t grow0 = (int64_t)rb * 128 + h * 32;
        uint32_t sc = 0;
        uint4 out;
        uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float x[16];
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint16_t mb = *reinterpret_cast<const uint16_t*>(cbase[i & 7] + (blk * 16 + i) * 128);  // tile row h*32+blk*16+i
            x[i] = __uint_as_float((uint32_t)mb << 16) - w[blk * 16 + i];
            amax = fmaxf(amax, fabsf(x[i]));
          }
          uint32_t code;
          const uint2 pk = quantize16(x, amax, g, rcp_table, p.rounding, p.seed, p.tag_col, p.step,
                                      (uint64_t)gcolj * (uint64_t)p.rows + (uint64_t)(grow0 + blk * 16), code);
          sc |= code << (8 * blk);
          o[2 * blk] = pk.x;
          o[2 * blk + 1] = pk.y;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[stage]);   // this warp is done with M
        *reinterpret_cast<uint4*>(p.col_codes + gcolj * (p.rows / 2) + grow0 / 2) = out;
        *reinterpret_cast<uint16_t*>(p.col_scales + scale_offset(gcolj, grow0 / 16, p.rows / 64)) = (uint16_t)sc;
      }
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// US (rows x KK) = U diag(S) and Vp (cols x KK) = V, zero-padded to KK columns.
__global__ void pad_factors_kernel(const float* __restrict__ U, const float* __restrict__ S,
                                   const float* __restrict__ V, int64_t rows, int64_t cols, int k, int KK,
                                   float* __restrict__ US, float* __restrict__ Vp) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nu = rows * KK;
  if (e < nu) {
    const int64_t i = e / KK;
    const int j = (int)(e - i * KK);
    US[e] = (j < k) ? U[i * k + j] * S[j] : 0.0f;
  } else if (e < nu + cols * KK) {
    const int64_t f = e - nu;
    const int64_t i = f / KK;
    const int j = (int)(f - i * KK);
    Vp[f] = (j < k) ? V[i * k + j] : 0.0f;
  }
}

bool map2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  EncodeTiledFn enc = encode_tiled();
  return enc && enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KK>
metis_status launch_kk(metis_ctx* ctx, const metis_matrix* M, const float* US, const float* Vp,
                       const metis_quant_params* q, const uint32_t* amax_bits, const metis_nvfp4* row,
                       const metis_nvfp4* col) {
  using C = RqCfg<KK>;
  CUtensorMap mM, mU, mV;
  if (!map2d(&mM, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, M->data, M->cols, M->rows, (uint64_t)M->ld * 2, 64, 128) ||
      !map2d(&mU, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, US, KK, M->rows, (uint64_t)KK * 4, 32, 128) ||
      !map2d(&mV, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Vp, KK, M->cols, (uint64_t)KK * 4, 32, 128))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed (residual quantization)");
  RqParams prm;
  prm.rows = M->rows;
  prm.cols = M->cols;
  prm.n_cb = (int)(M->cols / 128);
  prm.n_units = (int)((M->rows / 128) * prm.n_cb);
  prm.g = q->tensor_scale;
  prm.rounding = q->rounding;
  prm.seed = q->seed;
  prm.tag_row = stream_tag(q->operand_id, kPurposeSR, kSrRowwise);
  prm.tag_col = stream_tag(q->operand_id, kPurposeSR, kSrColwise);
  prm.step = q->step;
  prm.row_codes = row->codes;
  prm.row_scales = row->scales;
  prm.col_codes = col->codes;
  prm.col_scales = col->scales;
  prm.row_g = row->tensor_scale;
  prm.col_g = col->tensor_scale;
  prm.amax_bits = amax_bits;
  prm.status = ctx->status;
  auto kern = resquant_kernel<KK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(resquant)");
  const int grid = std::min(prm.n_units, ctx->sm_count);
  kern<<<grid, kRqThreads, C::SMEM, ctx->stream>>>(mM, mU, mV, prm); count_launch();
  return check_cuda(ctx, cudaGetLastError(), "resquant launch");
}

}  // namespace

metis_status run_residual_quantize(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                   const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col) {
  const int k = (f && f->k > 0) ? f->k : 0;
  const int KK = k <= 32 ? 32 : 64;
  const size_t need = (size_t)(M->rows + M->cols) * KK * 4 + 1024 + 256;
  metis_status s = ensure_workspace(ctx, need);
  if (s != METIS_OK) return s;
  Workspace ws{ctx->ws, ctx->ws_bytes};
  float* US = static_cast<float*>(ws.take((size_t)M->rows * KK * 4));
  float* Vp = static_cast<float*>(ws.take((size_t)M->cols * KK * 4));
  uint32_t* amax = nullptr;
  if (q->tensor_scale == 0.0f) {
    amax = static_cast<uint32_t*>(ws.take(256));
    if ((s = check_cuda(ctx, launch_amax(M->data, true, M->rows, M->cols, M->ld, amax, ctx->sm_count, ctx->stream),
                        "amax launch")) != METIS_OK)
      return s;
  }
  const int64_t n = (M->rows + M->cols) * KK;
  pad_factors_kernel<<<(unsigned)((n + 255) / 256), 256, 0, ctx->stream>>>(
      k ? f->U : nullptr, k ? f->S : nullptr, k ? f->V : nullptr, M->rows, M->cols, k, KK, US, Vp); count_launch();
  if ((s = check_cuda(ctx, cudaGetLastError(), "pad factors")) != METIS_OK) return s;
  return KK == 32 ? launch_kk<32>(ctx, M, US, Vp, q, amax, row, col) : launch_kk<64>(ctx, M, US, Vp, q, amax, row, col);
}

}  // namespace metis

namespace metis {

// Same work as run_residual_quantize, with the padded factor copies written to
// caller-provided device scratch of (rows + cols) * 64 floats instead of the
// context workspace.
metis_status run_residual_quantize_into(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                        const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col,
                                        float* scratch) {
  const int k = (f && f->k > 0) ? f->k : 0;
  const int KK = k <= 32 ? 32 : 64;
  float* US = scratch;
  float* Vp = scratch + M->rows * KK;
  uint32_t* amax = nullptr;
  metis_status s;
  if (q->tensor_scale == 0.0f) {
    amax = reinterpret_cast<uint32_t*>(scratch + kNoAllocAmaxOffset);
    if ((s = check_cuda(ctx, launch_amax(M->data, true, M->rows, M->cols, M->ld, amax, ctx->sm_count, ctx->stream),
                        "amax launch")) != METIS_OK)
      return s;
  }
  const int64_t n = (M->rows + M->cols) * KK;
  pad_factors_kernel<<<(unsigned)((n + 255) / 256), 256, 0, ctx->stream>>>(
      k ? f->U : nullptr, k ? f->S : nullptr, k ? f->V : nullptr, M->rows, M->cols, k, KK, US, Vp); count_launch();
  s = check_cuda(ctx, cudaGetLastError(), "pad factors");
  if (s != METIS_OK) return s;
  return KK == 32 ? launch_kk<32>(ctx, M, US, Vp, q, amax, row, col) : launch_kk<64>(ctx, M, US, Vp, q, amax, row, col);
}

}  // namespace metis
