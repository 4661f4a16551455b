// Fused residual + NVFP4 quantization in both orientations (one read of M).
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
// key design 1: M = U S V^T + M_R with the residual M_R quantized to NVFP4
// (background section: E2M1, 16-element blocks, E4M3 block scale; training
// strategy: stochastic rounding).  Every residual is quantized twice, with
// blocks along each GeMM contraction dimension that reads it.
//
// Reconstruction precision.  The notes write the split as exact, so the rank-k part
// U S V^T is rebuilt on the tensor cores to about 21 bits: every 128-row block of
// U diag(S) and of V is scaled by a power of two (largest entry in [2^14, 2^15)) and
// split into fp16 hi + lo, and the MMA accumulates hi*hi + hi*lo + lo*hi in fp32
// (the dropped lo*lo term and the two splits are each below 2^-22 of a product).  The
// residual is then one fp32 fused multiply-add, M + acc * (-2^-(a+b)), exact apart
// from its own rounding.
//
// Per 128 x 128 tile of M (persistent CTAs, contiguous row-block-major ranges):
//   warp 0      TMA: the scaled U S hi/lo rows of the row block (kept while the block
//               lasts), per tile the V hi/lo rows (2 stages) and the two 64-column
//               boxes of M (3 stages; 5 without factors)
//   warp 1      tensor-memory owner; one thread issues the twelve tcgen05.mma kind::f16
//               (M = N = 128, K = 16) of a tile into one of two fp32 accumulators
//   warps 2..17 a warp per 32 x 32 sub-tile (rows: its tensor-memory lane quarter):
//               residual of its rows from the accumulator and M, row-wise NVFP4 of
//               both 16-blocks of each row; the residual passes through the warp's own,
//               already read, 2 KB of the M stage as a transpose (two halves of 16
//               columns) and each lane quantizes one 16-row block of a column per half.
//               The warp stages its codes (1 KB) and writes them with two TMA stores;
//               its scales go straight to their 512-byte tiles.  The warps never wait
//               for one another.
// All mbarrier waits are bounded (METIS_DEV_TIMEOUT on expiry); on an abort the
// producer waits (bounded) for the tile loads it issued before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
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
constexpr int kSplitWidth = 64;                 // factor columns (k <= 64), zero-padded
constexpr long long kDrainLimitCycles = 20000000LL;   // ~10 ms: in-flight loads after an abort

template <bool kRecon>
struct RqCfg {
  static constexpr int A_BYTES = kRecon ? 32768 : 0;   // U S hi | lo: 2 boxes of 128 rows x 128 B
  static constexpr int V_BYTES = 32768;                // V hi | lo of the tile's 128 columns
  static constexpr int V_STAGES = kRecon ? 2 : 0;
  static constexpr int M_BYTES = 32768;                // two 64-column boxes of 16 KB
  static constexpr int M_STAGES = kRecon ? 3 : 5;
  static constexpr int OUT_BYTES = kRqEpiWarps * 1024;  // per warp: its row-wise then column-wise codes
  static constexpr int BAR_BYTES = 256;
  static constexpr int RCP_BYTES = 512;
  static constexpr size_t SMEM = 1024 + (size_t)A_BYTES + V_STAGES * V_BYTES + M_STAGES * M_BYTES + OUT_BYTES +
                                 BAR_BYTES + RCP_BYTES;
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
  const float* fac_a;          // 2^-a per 128-row block of U S (rows / 128)
  const float* fac_b;          // 2^-b per 128-row block of V (cols / 128)
  float* residual;             // non-null (parity surface): the fp32 residual, leading dimension ld_res
  int64_t ld_res;
  uint32_t* status;
  // Philox4x32-10 round keys of the SR stream (key = seed bumped by the Weyl constants),
  // read by the rounds straight from the parameter bank
  uint32_t rk0[10], rk1[10];
};

// fp16 x fp16 -> fp32, both operands K-major, M = N = 128.
constexpr uint32_t kIdescF16 = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(accumulate), "r"(kIdescF16)
      : "memory");
}

// ---- shared-memory accesses by 32-bit shared address ------------------------
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "r"(addr)
               : "memory");
  return r;
}
__device__ __forceinline__ uint4 lds_u32x4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr)
               : "memory");
  return r;
}

// ---- packed fp32 pairs (sm_100a) and the block maximum ----------------------
// d = a * s + c per lane, each an IEEE fused multiply-add rounded to nearest.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float s, float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rs, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rs, {%4, %4};\n\tmov.b64 rc, {%5, %6};\n\t"
      "fma.rn.f32x2 rd, ra, rs, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(s), "f"(c0), "f"(c1));
}
// d = a * s per lane, rounded to nearest.
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float s) {
  asm("{\n\t.reg .b64 ra, rs, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rs, {%4, %4};\n\t"
      "mul.rn.f32x2 rd, ra, rs;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(s));
}
// Largest of three magnitudes; NaN if any input is NaN.
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// max |x_i| over a 16-block (NaN if an element is NaN, Inf if one is infinite).
__device__ __forceinline__ float block_amax(const float* x) {
  const float m0 = max3_abs(x[0], x[1], x[2]);
  const float m1 = max3_abs(x[3], x[4], x[5]);
  const float m2 = max3_abs(x[6], x[7], x[8]);
  const float m3 = max3_abs(x[9], x[10], x[11]);
  const float m4 = max3_abs(x[12], x[13], x[14]);
  return max3_nan(max3_nan(m0, m1, m2), max3_nan(m3, m4, fabsf(x[15])), 0.0f);
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

// The four words of the SR stream's Philox4x32-10 call for counter (q, tag, step): the same
// generator as philox10() with the round keys taken from the kernel parameters and each
// 32 x 32 -> 64-bit product formed by one wide multiply.
__device__ __forceinline__ uint4 sr_words(const RqParams& p, uint32_t q, uint32_t tag) {
  uint32_t c0 = q, c1 = 0u, c2 = tag, c3 = p.step;   // counters below 2^32: rows * cols <= 2^36
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    uint64_t p0, p1;
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(p0) : "r"(0xD2511F53u), "r"(c0));
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(p1) : "r"(0xCD9E8D57u), "r"(c2));
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ p.rk0[r];
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ p.rk1[r];
    c0 = n0;
    c1 = (uint32_t)p1;
    c2 = n2;
    c3 = (uint32_t)p0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// One 16-element block with its maximum: scale code and packed codes (RN, or SR with the
// Philox call of counter qc = e0 / 16, e0 the index of the block's first element in the
// orientation's blocked order).
__device__ __forceinline__ uint2 quantize16(const RqParams& p, const float* v, float amax, float g,
                                            const float* rcp_table, uint32_t tag, uint32_t qc,
                                            uint32_t& scale_code) {
  const BlockScale bs = block_scale_fast(amax, g, rcp_table);
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) mul2(x[i], x[i + 1], v[i], v[i + 1], bs.rcp);
  uint2 packed;
  if (p.rounding) {
    const uint4 w = sr_words(p, qc, tag);
    packed.x = e2m1x4_sr(x[0], x[1], x[2], x[3], w.x) | (e2m1x4_sr(x[4], x[5], x[6], x[7], w.y) << 16);
    packed.y = e2m1x4_sr(x[8], x[9], x[10], x[11], w.z) | (e2m1x4_sr(x[12], x[13], x[14], x[15], w.w) << 16);
  } else {
    packed = encode_block16(x, 0, 0, 0, 0, 0);
  }
  if (bs.code == 0) packed = make_uint2(0, 0);
  scale_code = bs.code;
  return packed;
}

template <bool kRecon, bool kDump>
__global__ void __launch_bounds__(kRqThreads, 1)
    resquant_kernel(const __grid_constant__ CUtensorMap mapM, const __grid_constant__ CUtensorMap mapA,
                    const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapRowCodes,
                    const __grid_constant__ CUtensorMap mapColCodes, const RqParams p) {
  using C = RqCfg<kRecon>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sV = sA + C::A_BYTES;
  uint8_t* sM = sV + C::V_STAGES * C::V_BYTES;
  uint8_t* sOut = sM + C::M_STAGES * C::M_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + C::OUT_BYTES);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* v_full = bars + 2;                    // [2]
  uint64_t* v_empty = v_full + 2;                 // [2]
  uint64_t* m_full = v_empty + 2;                 // [M_STAGES <= 6]
  uint64_t* m_empty = m_full + 6;                 // [6]
  uint64_t* acc_full = m_empty + 6;               // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rcp_table = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::BAR_BYTES);   // 128 entries

  const float g = p.amax_bits ? auto_tensor_scale(*p.amax_bits) : p.g;
  for (int c = threadIdx.x; c < 128; c += blockDim.x)
    rcp_table[c] = c ? __frcp_rn(__fmul_rn(e4m3_value((uint32_t)c), g)) : 0.0f;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int u_begin = (int)(((int64_t)blockIdx.x * p.n_units) / gridDim.x);
  const int u_end = (int)(((int64_t)(blockIdx.x + 1) * p.n_units) / gridDim.x);

  if (threadIdx.x == 0) {
    tc::mbar_init(a_full, 1);
    tc::mbar_init(a_empty, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&v_full[s], 1);
      tc::mbar_init(&v_empty[s], 1);
      tc::mbar_init(&acc_full[s], 1);
      tc::mbar_init(&acc_empty[s], kRqEpiWarps);
    }
    for (int s = 0; s < C::M_STAGES; ++s) {
      tc::mbar_init(&m_full[s], 1);
      tc::mbar_init(&m_empty[s], kRqEpiWarps);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    if (blockIdx.x == 0) {
      *p.row_g = g;
      *p.col_g = g;
    }
  }
  if (kRecon && warp == 1) {   // two 128-column fp32 accumulators
    tc::tmem_alloc(tmem_slot, 256);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = kRecon ? *tmem_slot : 0u;

  auto fail_wait = [&]() {
    *abort_flag = 1;
    raise_status(p.status, METIS_DEV_TIMEOUT);
  };

  if (warp == 0) {
    if (lane == 0) {
      // parity of the last load issued into each slot (bit s), and which slots were used
      uint32_t m_par = 0, m_used = 0, v_par = 0, v_used = 0, a_par = 0, a_used = 0;
      int ms = 0, vs = 0;
      uint32_t mph = 0, vph = 0, aph = 0;
      int cur_rb = -1;
      for (int u = u_begin; u < u_end && !*abort_flag; ++u) {
        const int rb = u / p.n_cb, cb = u % p.n_cb;
        if (kRecon) {
          if (rb != cur_rb) {
            if (!tc::mbar_wait(a_empty, aph ^ 1u, abort_flag)) { fail_wait(); break; }
            tc::mbar_expect_tx(a_full, C::A_BYTES);
            tc::tma_load_2d(sA, &mapA, a_full, 0, rb * 128);
            tc::tma_load_2d(sA + 16384, &mapA, a_full, 64, rb * 128);
            a_par = aph;
            a_used = 1;
            aph ^= 1u;
            cur_rb = rb;
          }
          if (!tc::mbar_wait(&v_empty[vs], vph ^ 1u, abort_flag)) { fail_wait(); break; }
          uint8_t* dv = sV + vs * C::V_BYTES;
          tc::mbar_expect_tx(&v_full[vs], C::V_BYTES);
          tc::tma_load_2d(dv, &mapV, &v_full[vs], 0, cb * 128);
          tc::tma_load_2d(dv + 16384, &mapV, &v_full[vs], 64, cb * 128);
          v_par = (v_par & ~(1u << vs)) | (vph << vs);
          v_used |= 1u << vs;
          if (++vs == 2) {
            vs = 0;
            vph ^= 1u;
          }
        }
        if (!tc::mbar_wait(&m_empty[ms], mph ^ 1u, abort_flag)) { fail_wait(); break; }
        uint8_t* dm = sM + ms * C::M_BYTES;
        tc::mbar_expect_tx(&m_full[ms], C::M_BYTES);
        tc::tma_load_2d(dm, &mapM, &m_full[ms], cb * 128, rb * 128);
        tc::tma_load_2d(dm + 16384, &mapM, &m_full[ms], cb * 128 + 64, rb * 128);
        m_par = (m_par & ~(1u << ms)) | (mph << ms);
        m_used |= 1u << ms;
        if (++ms == C::M_STAGES) {
          ms = 0;
          mph ^= 1u;
        }
      }
      // No copy into this CTA's shared memory may still be in flight when it exits:
      // wait for the last phase issued on every slot (already complete unless aborted).
      for (int s = 0; s < C::M_STAGES; ++s)
        if (m_used >> s & 1u) tc::mbar_wait(&m_full[s], m_par >> s & 1u, nullptr, kDrainLimitCycles);
      for (int s = 0; s < 2; ++s)
        if (v_used >> s & 1u) tc::mbar_wait(&v_full[s], v_par >> s & 1u, nullptr, kDrainLimitCycles);
      if (a_used) tc::mbar_wait(a_full, a_par, nullptr, kDrainLimitCycles);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (kRecon && lane == 0) {
      int vs = 0;
      uint32_t vph = 0, aph = 0;
      int cur_rb = -1;
      int it = 0;
      for (int u = u_begin; u < u_end && !*abort_flag; ++u, ++it) {
        const int rb = u / p.n_cb;
        if (rb != cur_rb) {
          if (cur_rb >= 0) tc::tc_commit(a_empty);  // the old U S rows are no longer read
          if (!tc::mbar_wait(a_full, aph, abort_flag)) { fail_wait(); break; }
          aph ^= 1u;
          cur_rb = rb;
        }
        const int b = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!tc::mbar_wait(&v_full[vs], vph, abort_flag)) { fail_wait(); break; }
        if (!tc::mbar_wait(&acc_empty[b], (use & 1u) ^ 1u, abort_flag)) { fail_wait(); break; }
        tc::tc_fence_after();
        const uint8_t* v = sV + vs * C::V_BYTES;
        const uint64_t a_hi = tc::sdesc_sw128(tc::smem_addr(sA));
        const uint64_t a_lo = tc::sdesc_sw128(tc::smem_addr(sA + 16384));
        const uint64_t b_hi = tc::sdesc_sw128(tc::smem_addr(v));
        const uint64_t b_lo = tc::sdesc_sw128(tc::smem_addr(v + 16384));
        const uint32_t d = tmem + (uint32_t)(b * 128);
        // K = 64 in four steps of 16 halfs (32 bytes of the 128-byte swizzled rows)
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_f16(d, a_hi + 2 * j, b_hi + 2 * j, j ? 1u : 0u);
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_f16(d, a_hi + 2 * j, b_lo + 2 * j, 1u);
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_f16(d, a_lo + 2 * j, b_hi + 2 * j, 1u);
        tc::tc_commit(&v_empty[vs]);
        tc::tc_commit(&acc_full[b]);
        if (++vs == 2) {
          vs = 0;
          vph ^= 1u;
        }
      }
      tc::tc_commit(drain);
      tc::mbar_wait(drain, 0, nullptr, kDrainLimitCycles);
    }
    __syncwarp();
  } else {
    const int e = warp - 2;
    const int q = warp & 3;            // tensor-memory lane quarter: tile rows q*32 .. + 31
    const int h = e >> 2;              // tile columns h*32 .. + 31
    const int r = q * 32 + lane;       // tile row of this lane in the row pass
    const int jc = lane & 15;          // column (within a half) of this lane in the column pass
    const int hh = lane >> 4;          // 16-row half of the sub-tile in the column pass
    // The warp's own bytes of an M stage (rows q*32 .. + 31 of box h >> 1, its four 16-byte
    // chunks of each row) double as its transpose buffer once it has read them: element
    // (row l, column c) of a 32 x 16 half sits in row rho = q*32 + 8*(c & 3) + ((l >> 2) ^ (c & 7)),
    // chunk (h & 1)*4 + (c >> 2) (swizzled like M), word l & 3 -- conflict-free for the
    // 32 row-wise stores of a column and for the 128-bit loads of 16-row column blocks.
    const uint32_t box_off = (uint32_t)(h >> 1) * 16384;
    // Address parts of those accesses that depend on the lane only.  With S the (1024-byte
    // aligned) shared address of the stage's box, the fields below bit 10 combine by XOR:
    //   M row read, chunk j of the half:   (S + m_part) ^ (16 j)
    //   transpose store of column c:       ((S + t_part) ^ x(c)) + 1024 (c & 3)
    //   transpose load of chunk m4:         (S + l_part) ^ (144 m4)
    const uint32_t Kh = (uint32_t)(h & 1) * 4;
    const uint32_t L = (uint32_t)lane >> 2;
    const uint32_t m_part = (uint32_t)r * 128 + 16 * (Kh ^ ((uint32_t)r & 7));
    const uint32_t t_part = (uint32_t)q * 4096 + 128 * L + 16 * (Kh ^ L) + 4 * ((uint32_t)lane & 3);
    const uint32_t j7 = (uint32_t)jc & 7, k0 = 4 * (uint32_t)hh;
    const uint32_t l_part = (uint32_t)q * 4096 + 1024 * ((uint32_t)jc & 3) + 128 * (k0 ^ j7) +
                            16 * (Kh ^ ((uint32_t)jc >> 2) ^ k0 ^ j7);
    int ms = 0;
    uint32_t mph = 0;
    uint8_t* wout = sOut + e * 1024;   // this warp's staged codes: 32 rows x 16 B, then 32 columns x 16 B
    bool stored = false;               // a TMA store of this warp may still be reading wout
    // this lane's byte offsets in the scale tiles, less the tile's (row block, column block)
    // terms: the row-wise scale of (row r, block h) and the column-wise scales of (column
    // half * 16 + jc of this warp's 32, row block hh of its 32 rows)
    // (a 128-row block of the row-wise tiles spans cols / 64 tiles of 512 bytes: cols * 8)
    const int row_sc_lane = (h >> 1) * 512 + lane * 16 + q * 4 + 2 * (h & 1);
    const int col_sc_lane = (q >> 1) * 512 + jc * 16 + h * 4 + 2 * (q & 1) + hh;
    int rb = u_begin / p.n_cb, cb = u_begin % p.n_cb;   // the unit's 128-row and 128-column blocks
    for (int it = 0; it < u_end - u_begin; ++it, cb = cb + 1 == p.n_cb ? 0 : cb + 1, rb += cb == 0 ? 1 : 0) {
      const int b = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      bool ok = true;
      if (kRecon) ok = tc::mbar_wait(&acc_full[b], use & 1u, abort_flag);
      ok = ok && tc::mbar_wait(&m_full[ms], mph, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail_wait();
        break;
      }
      uint8_t* stage = sM + ms * C::M_BYTES;
      const uint32_t S = tc::smem_addr(stage) + box_off;
      const int64_t grow = (int64_t)rb * 128 + r;
      const int64_t gcol = (int64_t)cb * 128 + h * 32;
      const int64_t grow_t = (int64_t)rb * 128 + q * 32 + hh * 16;   // first row of this lane's column blocks
      // Philox counters (element index / 16) of the row-wise blocks of row r and of the
      // column-wise block of column gcol + jc; the second half adds 1 and rows respectively
      const uint32_t q_row = (uint32_t)grow * (uint32_t)(p.cols >> 4) + (uint32_t)(gcol >> 4);
      const uint32_t q_col = (uint32_t)(gcol + jc) * (uint32_t)(p.rows >> 4) + (uint32_t)(grow_t >> 4);
      float nf = 0.0f;
      if (kRecon) nf = -__fmul_rn(__ldg(p.fac_a + rb), __ldg(p.fac_b + cb));   // -2^-(a + b), exact
      uint4 row_out;
      uint32_t row_sc = 0;
      uint2 col_out[2];
      uint32_t col_sc[2];
      bool finite = true;
      // M row r, columns h*32 .. + 31: box h >> 1, chunks (h & 1)*4 .. + 3, all read before the
      // first transpose store reuses the region
      uint32_t mrow[16];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint4 raw = lds_u32x4((S + m_part) ^ (uint32_t)(16 * cc));
        mrow[4 * cc] = raw.x;
        mrow[4 * cc + 1] = raw.y;
        mrow[4 * cc + 2] = raw.z;
        mrow[4 * cc + 3] = raw.w;
      }
      __syncwarp();   // every lane has read its M row before the region is reused
      // the sub-tile in two halves of 16 columns: residual, row-wise block, transpose, column-wise block
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t* mw = mrow + 8 * half;
        float v[16];
        if (kRecon) {
          float acc[16];
          if (half == 0) tc::tc_fence_after();
          tc::tmem_load_16cols(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 128 + h * 32 + half * 16), acc);
          tc::tmem_load_wait();
          if (half == 1) {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[b]);   // both halves of the accumulator are read
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            fma2(v[2 * i], v[2 * i + 1], acc[2 * i], acc[2 * i + 1], nf, __uint_as_float(mw[i] << 16),
                 __uint_as_float(mw[i] & 0xFFFF0000u));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[2 * i] = __uint_as_float(mw[i] << 16);
            v[2 * i + 1] = __uint_as_float(mw[i] & 0xFFFF0000u);
          }
        }
        if (kDump) {
          float4* dst = reinterpret_cast<float4*>(p.residual + grow * p.ld_res + gcol + 16 * half);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        // transpose this half into the warp's region of the stage
        {
          const uint32_t T = S + t_part;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t x = 128u * (uint32_t)(c & 7) + 16u * ((uint32_t)(c >> 2) ^ (uint32_t)(c & 7));
            sts_f32((T ^ x) + 1024u * (uint32_t)(c & 3), v[c]);
          }
        }
        // row-wise block `half` of row r
        {
          const float amax = block_amax(v);
          finite &= amax <= 3.402823466e38f;   // false for NaN and Inf
          uint32_t code;
          const uint2 pk = quantize16(p, v, amax, g, rcp_table, p.tag_row, q_row + (uint32_t)half, code);
          row_sc |= code << (8 * half);
          if (half == 0) {
            row_out.x = pk.x;
            row_out.y = pk.y;
          } else {
            row_out.z = pk.x;
            row_out.w = pk.y;
          }
        }
        __syncwarp();
        // column-wise block: column half*16 + jc of the sub-tile, rows hh*16 .. + 15
        {
          float w[16];
#pragma unroll
          for (int m4 = 0; m4 < 4; ++m4) {
            const float4 t4 = lds_f32x4((S + l_part) ^ (144u * (uint32_t)m4));
            w[4 * m4] = t4.x;
            w[4 * m4 + 1] = t4.y;
            w[4 * m4 + 2] = t4.z;
            w[4 * m4 + 3] = t4.w;
          }
          const float amax = block_amax(w);
          col_out[half] = quantize16(p, w, amax, g, rcp_table, p.tag_col, q_col + (uint32_t)half * (uint32_t)p.rows,
                                     col_sc[half]);
        }
        __syncwarp();
      }
      if (lane == 0) tc::mbar_arrive(&m_empty[ms]);   // this warp is done with the M stage
      if (!finite) raise_status(p.status, METIS_DEV_NONFINITE);
      // ---- codes: staged per warp and written by two TMA stores (32 rows x 16 B each);
      // scales: straight to their 512-byte tiles (a warp's stores land in one tile)
      if (stored) {
        if (lane == 0) tc::bulk_wait_read_all();   // the previous tile's stores have read wout
        __syncwarp();
      }
      *reinterpret_cast<uint4*>(wout + lane * 16) = row_out;
#pragma unroll
      for (int half = 0; half < 2; ++half)
        *reinterpret_cast<uint2*>(wout + 512 + (half * 16 + jc) * 16 + hh * 8) = col_out[half];
      tc::fence_proxy_async();   // the staged bytes are read by the bulk-copy (async) proxy
      __syncwarp();
      if (lane == 0) {
        tc::tma_store_2d(&mapRowCodes, wout, cb * 64 + h * 16, rb * 128 + q * 32);
        tc::tma_store_2d(&mapColCodes, wout + 512, rb * 64 + q * 16, cb * 128 + h * 32);
        tc::bulk_commit_group();
      }
      stored = true;
      *reinterpret_cast<uint16_t*>(p.row_scales + (int64_t)rb * p.cols * 8 + (cb * 1024 + row_sc_lane)) =
          (uint16_t)row_sc;
#pragma unroll
      for (int half = 0; half < 2; ++half)
        p.col_scales[(int64_t)cb * p.rows * 8 + (rb * 1024 + col_sc_lane + half * 256)] = (uint8_t)col_sc[half];
      if (++ms == C::M_STAGES) {
        ms = 0;
        mph ^= 1u;
      }
    }
    if (lane == 0) tc::bulk_wait_all();   // no store may still read this CTA's shared memory at exit
  }

  tc::tc_fence_before();
  __syncthreads();
  if (kRecon && warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

// One CTA per 128-row block of U diag(S) (the first rows / 128 CTAs) or of V (the rest):
// the block's largest |entry| m sets the power of two 2^e with m 2^e in [2^14, 2^15)
// (e kept in [-63, 63]; 0 for an all-zero block), and every entry x (k columns, padded
// with zeros to 64) is written as the fp16 pair hi = RN16(x 2^e), lo = RN16(x 2^e - hi):
// row i of the output holds the 64 hi values, then the 64 lo values.  fac[block] = 2^-e.
// A block of 512 threads holds its 128 x 64 tile in registers -- four runs of four
// consecutive columns a thread, loaded as float4 when k = 64 and the factors are 16-byte
// aligned -- reduces the maximum, then writes each run's four hi and four lo values as
// one 8-byte store each.
constexpr int kSplitFacThreads = 512;
constexpr int kSplitFacRuns = 128 * kSplitWidth / 4 / kSplitFacThreads;
__global__ void __launch_bounds__(kSplitFacThreads) split_factors_kernel(
    const float* __restrict__ U, const float* __restrict__ S, const float* __restrict__ V, int64_t rows, int k,
    bool vec, __half* __restrict__ A16, __half* __restrict__ B16, float* __restrict__ fac_a,
    float* __restrict__ fac_b) {
  __shared__ float red[kSplitFacThreads / 32];
  const int64_t nb_a = rows / 128;
  const bool is_a = (int64_t)blockIdx.x < nb_a;
  const int64_t blk = is_a ? (int64_t)blockIdx.x : (int64_t)blockIdx.x - nb_a;
  const float* F = (is_a ? U : V) + blk * 128 * k;
  __half* out = (is_a ? A16 : B16) + blk * 128 * 128;
  float v[kSplitFacRuns][4];
#pragma unroll
  for (int it = 0; it < kSplitFacRuns; ++it) {
    const int t = threadIdx.x + it * kSplitFacThreads;
    const int i = t >> 4, j0 = (t & 15) * 4;
    if (vec) {
      const float4 x = *reinterpret_cast<const float4*>(F + i * kSplitWidth + j0);
      v[it][0] = x.x;
      v[it][1] = x.y;
      v[it][2] = x.z;
      v[it][3] = x.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[it][e] = j0 + e < k ? F[i * k + j0 + e] : 0.0f;
    }
  }
  float m = 0.0f;
#pragma unroll
  for (int it = 0; it < kSplitFacRuns; ++it) {
    const int j0 = ((threadIdx.x + it * kSplitFacThreads) & 15) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (is_a) v[it][e] = j0 + e < k ? __fmul_rn(v[it][e], S[j0 + e]) : 0.0f;
      m = fmaxf(m, fabsf(v[it][e]));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < kSplitFacThreads / 32; ++w) m = fmaxf(m, red[w]);
  int ex = 0;
  if (m > 0.0f && m <= 3.402823466e38f) {
    const int fl = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;   // floor(log2 m); -127 for subnormal m
    ex = min(63, max(-63, 14 - fl));
  }
  const float up = __uint_as_float((uint32_t)(ex + 127) << 23);
  if (threadIdx.x == 0) (is_a ? fac_a : fac_b)[blk] = __uint_as_float((uint32_t)(127 - ex) << 23);
#pragma unroll
  for (int it = 0; it < kSplitFacRuns; ++it) {
    const int t = threadIdx.x + it * kSplitFacThreads;
    const int i = t >> 4, j0 = (t & 15) * 4;
    __half hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x = __fmul_rn(v[it][e], up);
      hi[e] = __float2half_rn(x);
      lo[e] = __float2half_rn(__fsub_rn(x, __half2float(hi[e])));
    }
    *reinterpret_cast<uint2*>(out + i * 128 + j0) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(out + i * 128 + 64 + j0) = *reinterpret_cast<const uint2*>(lo);
  }
}

bool map2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  EncodeTiledFn enc = encode_tiled();
  return enc && enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kRecon, bool kDump>
metis_status launch_rq(metis_ctx* ctx, const metis_matrix* M, const CUtensorMap& mA, const CUtensorMap& mV,
                       RqParams prm) {
  using C = RqCfg<kRecon>;
  CUtensorMap mM, mRow, mCol;
  if (!map2d(&mM, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, M->data, M->cols, M->rows, (uint64_t)M->ld * 2, 64, 128) ||
      !map2d(&mRow, CU_TENSOR_MAP_DATA_TYPE_UINT8, prm.row_codes, M->cols / 2, M->rows, M->cols / 2, 16, 32,
             CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !map2d(&mCol, CU_TENSOR_MAP_DATA_TYPE_UINT8, prm.col_codes, M->rows / 2, M->cols, M->rows / 2, 16, 32,
             CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed (residual quantization)");
  auto kern = resquant_kernel<kRecon, kDump>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(resquant)");
  const int grid = std::min(prm.n_units, ctx->sm_count);
  const bool prof = ctx->profiling && !kDump;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  if (prof) {
    cudaEventCreate(&ev0);
    cudaEventCreate(&ev1);
    cudaEventRecord(ev0, ctx->stream);
  }
  kern<<<grid, kRqThreads, C::SMEM, ctx->stream>>>(mM, mA, mV, mRow, mCol, prm); count_launch();
  if (prof) {
    cudaEventRecord(ev1, ctx->stream);
    // algorithmic bytes: 2 B read and 2 x (1/2 + 1/16) B written per element
    profile_record(ctx, kProfResquant, ev0, ev1, 3.125 * (double)M->rows * (double)M->cols);
  }
  return check_cuda(ctx, cudaGetLastError(), "resquant launch");
}

}  // namespace

// Scratch layout (bytes from `scratch`, 256-byte aligned pieces):
//   A16 rows x 128 fp16, B16 cols x 128 fp16, fac_a rows / 128 floats, fac_b cols / 128 floats.
size_t residual_quantize_scratch_bytes(int64_t rows, int64_t cols) {
  const auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  return up((size_t)rows * 256) + up((size_t)cols * 256) + up((size_t)rows / 128 * 4) + up((size_t)cols / 128 * 4);
}

metis_status run_residual_quantize_into(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                        const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col,
                                        void* scratch, uint32_t* amax_word, float* residual, int64_t ld_res) {
  const int k = (f && f->k > 0) ? f->k : 0;
  const bool recon = k > 0;
  metis_status s;
  Workspace ws{static_cast<char*>(scratch), residual_quantize_scratch_bytes(M->rows, M->cols)};
  __half* A16 = static_cast<__half*>(ws.take((size_t)M->rows * 256));
  __half* B16 = static_cast<__half*>(ws.take((size_t)M->cols * 256));
  float* fac_a = static_cast<float*>(ws.take((size_t)M->rows / 128 * 4));
  float* fac_b = static_cast<float*>(ws.take((size_t)M->cols / 128 * 4));
  uint32_t* amax = nullptr;
  if (q->tensor_scale == 0.0f) {
    amax = amax_word;
    if ((s = check_cuda(ctx, launch_amax(M->data, true, M->rows, M->cols, M->ld, amax, ctx->sm_count, ctx->stream),
                        "amax launch")) != METIS_OK)
      return s;
  }
  CUtensorMap mA, mV;
  if (recon) {
    const unsigned nblk = (unsigned)(M->rows / 128 + M->cols / 128);
    const bool vec = k == kSplitWidth && reinterpret_cast<uintptr_t>(f->U) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(f->V) % 16 == 0;
    split_factors_kernel<<<nblk, kSplitFacThreads, 0, ctx->stream>>>(f->U, f->S, f->V, M->rows, k, vec, A16, B16,
                                                                     fac_a, fac_b);
    count_launch();
    if ((s = check_cuda(ctx, cudaGetLastError(), "split factors")) != METIS_OK) return s;
    if (!map2d(&mA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, A16, 128, M->rows, 256, 64, 128) ||
        !map2d(&mV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, B16, 128, M->cols, 256, 64, 128))
      return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed (factor tiles)");
  } else {
    mA = mV = CUtensorMap{};
  }
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
  prm.amax_bits = amax;
  prm.fac_a = fac_a;
  prm.fac_b = fac_b;
  prm.residual = residual;
  prm.ld_res = ld_res;
  prm.status = ctx->status;
  for (int r = 0; r < 10; ++r) {   // Weyl-sequence round keys of Philox4x32-10
    prm.rk0[r] = (uint32_t)q->seed + (uint32_t)r * 0x9E3779B9u;
    prm.rk1[r] = (uint32_t)(q->seed >> 32) + (uint32_t)r * 0xBB67AE85u;
  }
  if (residual)
    return recon ? launch_rq<true, true>(ctx, M, mA, mV, prm) : launch_rq<false, true>(ctx, M, mA, mV, prm);
  return recon ? launch_rq<true, false>(ctx, M, mA, mV, prm) : launch_rq<false, false>(ctx, M, mA, mV, prm);
}

metis_status run_residual_quantize(metis_ctx* ctx, const metis_matrix* M, const metis_factors* f,
                                   const metis_quant_params* q, const metis_nvfp4* row, const metis_nvfp4* col,
                                   float* residual, int64_t ld_res) {
  const size_t bytes = residual_quantize_scratch_bytes(M->rows, M->cols);
  metis_status s = ensure_workspace(ctx, bytes + 256);
  if (s != METIS_OK) return s;
  return run_residual_quantize_into(ctx, M, f, q, row, col, ctx->ws, reinterpret_cast<uint32_t*>(ctx->ws + bytes),
                                    residual, ld_res);
}

}  // namespace metis
