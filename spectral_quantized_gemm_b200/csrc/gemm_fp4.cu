// Block-scaled NVFP4 GeMM on the sm_100a tensor cores, with the Metis rank-fold.
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
// key design 1.  Expanding the forward equation around the residual product,
//   (L_A S_A R_A^T + A_R)(L_B S_B R_B^T + B_R)
//     = A_R B_R + [L_A | T_B] [T_A ; R_B^T],
//   T_A = S_A R_A^T (B_R + L_B S_B R_B^T),   T_B = A_R L_B S_B,
// so every GeMM of the layer is one FP4 x FP4 product plus a rank-2k bf16
// product.  This kernel runs both into the same fp32 tensor-memory accumulator:
// the K loop streams NVFP4 stages (tcgen05 kind::mxf4nvf4, block16 UE4M3 scales)
// and then the fold stages (kind::f16, bf16 operands) through one shared-memory
// ring, and the epilogue scales by alpha (and an optional per-column factor).
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A/B tiles (128-byte swizzle), scale tiles (bulk copy)
//   warp 1      tensor-memory owner and MMA issuer (one thread)
//   warps 2..9  epilogue: tcgen05.ld of the accumulator, scale, store
//   warps 10-11 scale copies (shared -> tensor memory) of each stage, split between
//               two issuing threads: issued from the MMA thread they serialized with
//               the MMAs and cost about a quarter of the kernel's time
// Every mbarrier wait is bounded; on expiry the CTA raises METIS_DEV_TIMEOUT,
// stops issuing work and exits after releasing its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace metis {
namespace {

constexpr int kThreads = 384;
constexpr int kEpiWarps = 8;

template <int BN>
struct Cfg {
  static constexpr int BM = 128;
  static constexpr int A_BYTES = BM * 128;                // one 128-byte swizzle row per matrix row
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFB_ATOMS = BN > 128 ? 2 : 1;      // 128-row scale tiles of B
  static constexpr int SFA_BYTES = 4 * 512;               // 4 k-tiles of 64 per 256-element stage
  static constexpr int SFB_BYTES = SFB_ATOMS * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = BN > 128 ? 4 : (BN == 128 ? 6 : 6);
  static constexpr int SFB_COLS_PER_K = SFB_ATOMS * 4;
  // scale columns of one stage: SFA (4 per MMA k-step) then SFB
  static constexpr int SF_SET_COLS = 16 + 4 * SFB_COLS_PER_K;
  // two accumulator buffers (epilogue of tile t overlaps the MMAs of tile t+1)
  // whenever they fit next to two sets of scale columns in the 512 tensor-memory columns
  static constexpr int ACC_BUFS = (2 * BN + 2 * SF_SET_COLS) <= 512 ? 2 : 1;
  static constexpr int ACC_COLS = BN * ACC_BUFS;
  // one set of scale columns per ring stage, so the copy of stage s + 1's scales never
  // waits for the MMAs of stage s to finish reading theirs
  static constexpr int SF_SETS = STAGES;
  static constexpr int USED_COLS = ACC_COLS + SF_SETS * SF_SET_COLS;
  static constexpr int TMEM_COLS = USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64 : USED_COLS <= 128 ? 128
                                   : USED_COLS <= 256 ? 256 : 512;
  // ring, barriers, then one 1 KB store-staging buffer per epilogue warp
  static constexpr size_t SMEM = (size_t)STAGES * (STAGE_BYTES + SF_STAGE_BYTES) + 1024 + 256 + kEpiWarps * 1024;
  static_assert(USED_COLS <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  const uint8_t* sfa;
  const uint8_t* sfb;
  int64_t kb_tiles;  // K / 64: scale tiles per 128-row block
  const float* ga;
  const float* gb;
  float alpha_extra;
  const float* col_scale;
  void* C;
  int64_t ldc;
  int c_dtype;
  int m_tiles, n_tiles;
  int k_stages, fold_stages;
  int k_splits;            // work units per output tile along K (split-K), >= 1
  int64_t split_stride;    // elements between the partial outputs of consecutive splits
  uint32_t* status;
  // Grouped launch (thin GeMMs only): after the units of the problem above come the units
  // of n_extra more problems with their own operands (maps A1/B1, A2/B2), scales, tensor
  // scales, fp32 output and tiling; one column tile each, the same K, no fold stages.
  int n_extra;
  struct Extra {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* ga;
    const float* gb;
    float* C;
    int64_t ldc;
    int m_tiles, k_splits;
    int64_t split_stride;
  } extra[2];
};

// Where a work unit of a (possibly grouped) launch lands: problem g, output tile
// (mb, nb), K-stage range [s0, s1), split index.
struct Unit {
  int g, mb, nb, s0, s1, split;
};

__device__ __forceinline__ Unit decode_unit(const Params& p, int unit, int total_stages) {
  int g = 0, m_tiles = p.m_tiles, n_tiles = p.n_tiles, splits = p.k_splits;
  int u = unit;
  int units = m_tiles * n_tiles * splits;
  for (int e = 0; e < p.n_extra && u >= units; ++e) {
    u -= units;
    g = e + 1;
    m_tiles = p.extra[e].m_tiles;
    n_tiles = 1;
    splits = p.extra[e].k_splits;
    units = m_tiles * splits;
  }
  Unit r;
  const int num_tiles = m_tiles * n_tiles;
  const int tile = u % num_tiles;
  const int per = (total_stages + splits - 1) / splits;
  r.g = g;
  r.mb = tile % m_tiles;
  r.nb = tile / m_tiles;
  r.split = u / num_tiles;
  r.s0 = r.split * per;
  r.s1 = min(total_stages, r.s0 + per);
  return r;
}

// Output of one problem of a launch.
struct OutView {
  void* C;
  int64_t ldc;
  int c_dtype;
  const float* col_scale;
};

// Epilogue store of one warp's 32-row slice: lane t holds row row0 + t, columns
// [cbase, cbase + COLS) in v.  Chunks of 32 bytes per row (16 bf16 or 8 fp32 columns) go
// through the warp's 1 KB staging buffer and leave as full 32-byte sectors: lane pairs
// store the two halves of one row, 16 rows per instruction.  (Storing each lane's own
// row directly wrote half sectors and cost a fifth of the GeMM's time.)  fp32 output
// goes to f32_out (a split-K partial or C); bf16 output to C.
template <int COLS>
__device__ __forceinline__ void store_rows(const OutView& p, const float (&v)[COLS], uint8_t* buf, int lane,
                                           int64_t row0, int64_t cbase, float alpha, float* f32_out) {
  uint4* stage_buf = reinterpret_cast<uint4*>(buf);
  const int half = lane & 1;
  if (p.c_dtype == METIS_OUT_F32) {
#pragma unroll
    for (int c = 0; c < COLS; c += 8) {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = v[c + i] * alpha * (p.col_scale ? p.col_scale[cbase + c + i] : 1.0f);
      stage_buf[lane * 2] = make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                                       __float_as_uint(o[3]));
      stage_buf[lane * 2 + 1] = make_uint4(__float_as_uint(o[4]), __float_as_uint(o[5]), __float_as_uint(o[6]),
                                           __float_as_uint(o[7]));
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int r = (lane >> 1) + 16 * t;
        float* dst = f32_out + (row0 + r) * p.ldc + cbase + c + half * 4;
        *reinterpret_cast<uint4*>(dst) = stage_buf[r * 2 + half];
      }
      __syncwarp();
    }
  } else {
    __nv_bfloat16* const out = reinterpret_cast<__nv_bfloat16*>(p.C);
#pragma unroll
    for (int c = 0; c < COLS; c += 16) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = v[c + 2 * i] * alpha * (p.col_scale ? p.col_scale[cbase + c + 2 * i] : 1.0f);
        const float b = v[c + 2 * i + 1] * alpha * (p.col_scale ? p.col_scale[cbase + c + 2 * i + 1] : 1.0f);
        const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
        w[i] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      stage_buf[lane * 2] = make_uint4(w[0], w[1], w[2], w[3]);
      stage_buf[lane * 2 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int r = (lane >> 1) + 16 * t;
        __nv_bfloat16* dst = out + (row0 + r) * p.ldc + cbase + c + half * 8;
        *reinterpret_cast<uint4*>(dst) = stage_buf[r * 2 + half];
      }
      __syncwarp();
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                      const __grid_constant__ CUtensorMap mapFa, const __grid_constant__ CUtensorMap mapFb,
                      const __grid_constant__ CUtensorMap mapA1, const __grid_constant__ CUtensorMap mapB1,
                      const __grid_constant__ CUtensorMap mapA2, const __grid_constant__ CUtensorMap mapB2,
                      const Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* sf = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sf + C::STAGES * C::SF_STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tmem_full = bars + 2 * C::STAGES;   // [2]
  uint64_t* tmem_empty = tmem_full + 2;         // [2]
  uint64_t* drain = tmem_full + 4;
  uint64_t* sf_ready = tmem_full + 5;           // [STAGES] the stage's scales are in tensor memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_ready + C::STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* epi_smem = reinterpret_cast<uint8_t*>(bars) + 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
      tc::mbar_init(&sf_ready[s], 2);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tmem_full[b], 1);
      tc::mbar_init(&tmem_empty[b], kEpiWarps);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&mapA);
    tc::prefetch_tensormap(&mapB);
    if (p.fold_stages) {
      tc::prefetch_tensormap(&mapFa);
      tc::prefetch_tensormap(&mapFb);
    }
    if (p.n_extra > 0) {
      tc::prefetch_tensormap(&mapA1);
      tc::prefetch_tensormap(&mapB1);
    }
    if (p.n_extra > 1) {
      tc::prefetch_tensormap(&mapA2);
      tc::prefetch_tensormap(&mapB2);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total_stages = p.k_stages + p.fold_stages;
  int num_units = p.m_tiles * p.n_tiles * p.k_splits;
  for (int e = 0; e < p.n_extra; ++e) num_units += p.extra[e].m_tiles * p.extra[e].k_splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int unit = blockIdx.x; unit < num_units && !*abort_flag; unit += gridDim.x) {
        const Unit w = decode_unit(p, unit, total_stages);
        const int mb = w.mb, nb = w.nb;
        const CUtensorMap* mA = w.g == 0 ? &mapA : (w.g == 1 ? &mapA1 : &mapA2);
        const CUtensorMap* mB = w.g == 0 ? &mapB : (w.g == 1 ? &mapB1 : &mapB2);
        const uint8_t* sfa_g = w.g == 0 ? p.sfa : p.extra[w.g - 1].sfa;
        const uint8_t* sfb_g = w.g == 0 ? p.sfb : p.extra[w.g - 1].sfb;
        for (int kk = w.s0; kk < w.s1; ++kk) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          uint8_t* sA = tiles + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          if (kk < p.k_stages) {
            uint8_t* sSFA = sf + stage * C::SF_STAGE_BYTES;
            uint8_t* sSFB = sSFA + C::SFA_BYTES;
            tc::mbar_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + C::SFA_BYTES + C::SFB_BYTES);
            tc::tma_load_2d(sA, mA, &full[stage], kk * 128, mb * 128);
            tc::tma_load_2d(sB, mB, &full[stage], kk * 128, nb * BN);
            tc::bulk_load(sSFA, sfa_g + ((int64_t)mb * p.kb_tiles + kk * 4) * 512, C::SFA_BYTES, &full[stage]);
            const int64_t nb128 = (int64_t)nb * BN / 128;
#pragma unroll
            for (int a = 0; a < C::SFB_ATOMS; ++a)
              tc::bulk_load(sSFB + a * 2048, sfb_g + ((nb128 + a) * p.kb_tiles + kk * 4) * 512, 2048,
                            &full[stage]);
          } else {
            const int f = kk - p.k_stages;
            tc::mbar_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
            tc::tma_load_2d(sA, &mapFa, &full[stage], f * 64, mb * 128);
            tc::tma_load_2d(sB, &mapFb, &full[stage], f * 64, nb * BN);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t id_fp4 = tc::idesc_nvf4(BN);
      const uint32_t id_bf16 = tc::idesc_bf16(BN);

      for (int unit = blockIdx.x; unit < num_units && !*abort_flag; unit += gridDim.x, ++it) {
        const Unit w = decode_unit(p, unit, total_stages);
        const int s0 = w.s0, s1 = w.s1;
        const int ab = it % C::ACC_BUFS;
        const uint32_t use = (uint32_t)(it / C::ACC_BUFS);
        const uint32_t t_acc = tmem + ab * BN;
        if (!tc::mbar_wait(&tmem_empty[ab], (use & 1u) ^ 1u, abort_flag)) {
          *abort_flag = 1;
          raise_status(p.status, METIS_DEV_TIMEOUT);
          break;
        }
        tc::tc_fence_after();
        for (int kk = s0; kk < s1; ++kk) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag) ||
              !tc::mbar_wait(&sf_ready[stage], phase, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          tc::tc_fence_after();
          const uint8_t* sA = tiles + stage * C::STAGE_BYTES;
          const uint8_t* sB = sA + C::A_BYTES;
          const uint64_t adesc = tc::sdesc_sw128(tc::smem_addr(sA));
          const uint64_t bdesc = tc::sdesc_sw128(tc::smem_addr(sB));
          if (kk < p.k_stages) {
            const uint32_t t_sfa = tmem + C::ACC_COLS + stage * C::SF_SET_COLS;
            const uint32_t t_sfb = t_sfa + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc::mma_nvf4(t_acc, adesc + 2 * j, bdesc + 2 * j, id_fp4, t_sfa + 4 * j,
                           t_sfb + C::SFB_COLS_PER_K * j, (kk != s0 || j) ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc::mma_bf16(t_acc, adesc + 2 * j, bdesc + 2 * j, id_bf16, (kk != s0 || j) ? 1u : 0u);
          }
          tc::tc_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (*abort_flag) break;
        tc::tc_commit(&tmem_full[ab]);
      }
      // let every issued tensor-core operation finish before the memory is released
      tc::tc_commit(drain);
      tc::mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ scale copies
    // Thread 0 of warp 10 copies SFA of k-steps 0-1 and the first 128-row atom of SFB,
    // thread 0 of warp 11 SFA of k-steps 2-3 and the second SFB atom (six copies each
    // for N = 256); both commit to the stage's sf_ready (count 2), for fold stages too,
    // so its phases follow the ring.  A stage's scale columns are free again once the
    // stage is refilled (its previous MMAs committed empty).
    const int part = warp - 10;
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int unit = blockIdx.x; unit < num_units && !*abort_flag; unit += gridDim.x) {
        const Unit w = decode_unit(p, unit, total_stages);
        for (int kk = w.s0; kk < w.s1; ++kk) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          tc::tc_fence_after();
          if (kk < p.k_stages) {
            const uint8_t* sSFA = sf + stage * C::SF_STAGE_BYTES;
            const uint8_t* sSFB = sSFA + C::SFA_BYTES;
            const uint32_t t_sfa = tmem + C::ACC_COLS + stage * C::SF_SET_COLS;
            const uint32_t t_sfb = t_sfa + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if ((j >> 1) == part)
                tc::tc_copy_32x128b_x4(t_sfa + 4 * j, tc::sdesc_scales(tc::smem_addr(sSFA + 512 * j)));
#pragma unroll
              for (int a = 0; a < C::SFB_ATOMS; ++a)
                if (a == part || (C::SFB_ATOMS == 1 && part == 0))
                  tc::tc_copy_32x128b_x4(t_sfb + C::SFB_COLS_PER_K * j + 4 * a,
                                         tc::sdesc_scales(tc::smem_addr(sSFB + 2048 * a + 512 * j)));
            }
          }
          tc::tc_commit(&sf_ready[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // tensor-memory lane quarter of this warp
    const int h = (warp - 2) >> 2;          // column half
    constexpr int kColsPerWarp = BN >= 64 ? BN / 2 : BN;
    const bool active = BN >= 64 || h == 0;
    int it = 0;
    for (int unit = blockIdx.x; unit < num_units; unit += gridDim.x, ++it) {
      const Unit w = decode_unit(p, unit, total_stages);
      const int ab = it % C::ACC_BUFS;
      const uint32_t use = (uint32_t)(it / C::ACC_BUFS);
      OutView ov{p.C, p.ldc, p.c_dtype, p.col_scale};
      float alpha = (p.ga ? *p.ga : 1.0f) * (p.gb ? *p.gb : 1.0f) * p.alpha_extra;
      int64_t split_stride = p.split_stride;
      if (w.g > 0) {
        const Params::Extra& x = p.extra[w.g - 1];
        ov = OutView{x.C, x.ldc, METIS_OUT_F32, nullptr};
        alpha = (x.ga ? *x.ga : 1.0f) * (x.gb ? *x.gb : 1.0f);
        split_stride = x.split_stride;
      }
      float* const split_out = reinterpret_cast<float*>(ov.C) + (int64_t)w.split * split_stride;
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&tmem_full[ab], use & 1u, abort_flag));
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          raise_status(p.status, METIS_DEV_TIMEOUT);
        }
        break;
      }
      tc::tc_fence_after();
      const int mb = w.mb, nb = w.nb;
      float v[kColsPerWarp];
      const int col0 = active ? h * kColsPerWarp : 0;
      if (active) {
#pragma unroll
        for (int c = 0; c < kColsPerWarp; c += 16) {
          float t[16];
          uint32_t r[16];
          const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * BN + col0 + c);
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
              "%13, %14, %15}, [%16];"
              : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                "=r"(r[15])
              : "r"(taddr));
#pragma unroll
          for (int i = 0; i < 16; ++i) t[i] = __uint_as_float(r[i]);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[c + i] = t[i];
        }
        tc::tmem_load_wait();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tmem_empty[ab]);
      if (active)
        store_rows(ov, v, epi_smem + (warp - 2) * 1024, lane, (int64_t)mb * 128 + q * 32, (int64_t)nb * BN + col0,
                   alpha, split_out);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
// The large GeMMs (both output dimensions multiples of 256, no split-K) run on CTA
// pairs: a cluster of two CTAs computes a 256 x 256 output tile with cta_group::2 MMAs
// (M = 256, N = 256).  Each CTA loads its own 128 rows of A, its 128 rows of B, the
// scales of its A rows and of all 256 B rows: 38 KB per K stage for the MMA work that
// takes 54 KB in a single-CTA 128 x 256 tile, and each MMA reads half of B from the
// other SM's shared memory.
//   both CTAs, warp 0: TMA loads of the CTA's tiles; the bytes are counted on the even
//     CTA's stage barrier, so the even CTA learns that the whole pair stage landed
//   even CTA, warp 1: the pair-wide MMAs; commits free the stage in both CTAs and hand
//     each CTA its accumulator
//   even CTA, warps 10-11: pair-wide block-scale copies (each CTA's scales into its own
//     tensor memory), committed to the stage's sf_ready barrier
//   both CTAs, warps 2-9: epilogue of the CTA's own 128 rows; the drain is reported to
//     the even CTA's accumulator-empty barrier
// Waits are bounded as in the single-CTA kernel, and both CTAs always reach the final
// cluster barrier before the tensor memory is released.
struct PairCfg {
  static constexpr int BN = 256;
  static constexpr int A_BYTES = 128 * 128;        // this CTA's 128 rows, 256 K elements
  static constexpr int B_BYTES = 128 * 128;        // this CTA's 128 of the 256 B rows
  static constexpr int SFA_BYTES = 4 * 512;        // scales of this CTA's A rows
  static constexpr int SFB_BYTES = 2 * 4 * 512;    // scales of all 256 B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = 5;
  static constexpr int SFB_COLS_PER_K = 8;
  static constexpr int SF_SET_COLS = 16 + 4 * SFB_COLS_PER_K;
  static constexpr int ACC_COLS = 256;
  static constexpr int USED_COLS = ACC_COLS + STAGES * SF_SET_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t PAIR_TX = 2 * (STAGE_BYTES + SF_STAGE_BYTES);  // an NVFP4 stage of the pair
  static constexpr uint32_t PAIR_FOLD_TX = 2 * STAGE_BYTES;               // a bf16 fold stage of the pair
  // output staging: per epilogue warp one 128-byte-swizzled box of 32 rows x 128 bytes
  static constexpr int EPI_WARP_BYTES = 4096;
  static constexpr size_t SMEM =
      (size_t)STAGES * (STAGE_BYTES + SF_STAGE_BYTES) + kEpiWarps * EPI_WARP_BYTES + 1024 + 256;
  static_assert(USED_COLS <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                           const __grid_constant__ CUtensorMap mapFa, const __grid_constant__ CUtensorMap mapFb,
                           const __grid_constant__ CUtensorMap mapSa, const __grid_constant__ CUtensorMap mapSb,
                           const __grid_constant__ CUtensorMap mapC, const Params p) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* sf = smem + C::STAGES * C::STAGE_BYTES;
  uint8_t* epi = sf + C::STAGES * C::SF_STAGE_BYTES;   // 1024-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + kEpiWarps * C::EPI_WARP_BYTES);
  uint64_t* full = bars;                          // (even CTA) the pair's stage landed
  uint64_t* empty = bars + C::STAGES;             // the pair's MMAs are done with the stage
  uint64_t* sf_ready = bars + 2 * C::STAGES;      // (even CTA) the stage's scales are in tensor memory
  uint64_t* tmem_full = bars + 3 * C::STAGES;     // this CTA's accumulator is complete
  uint64_t* tmem_empty = tmem_full + 1;           // (even CTA) both CTAs' epilogues drained
  uint64_t* drain = tmem_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const bool even = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
      tc::mbar_init(&sf_ready[s], 2);
    }
    tc::mbar_init(tmem_full, 1);
    tc::mbar_init(tmem_empty, 2 * kEpiWarps);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&mapA);
    tc::prefetch_tensormap(&mapB);
    tc::prefetch_tensormap(&mapSa);
    tc::prefetch_tensormap(&mapSb);
    tc::prefetch_tensormap(&mapC);
    if (p.fold_stages) {
      tc::prefetch_tensormap(&mapFa);
      tc::prefetch_tensormap(&mapFb);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish_pair();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();   // both CTAs' barriers exist before any cross-CTA arrival
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_tiles = p.m_tiles * p.n_tiles;   // m_tiles counts 256-row blocks
  const int total_stages = p.k_stages + p.fold_stages;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0 = tc::cluster_addr(&full[0], 0);   // the even CTA's stage barriers
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < num_tiles && !*abort_flag; tile += npairs) {
        const int mb = tile % p.m_tiles;
        const int nb = tile / p.m_tiles;
        const int arow = mb * 256 + (int)rank * 128;
        const int brow = nb * C::BN + (int)rank * 128;
        for (int kk = 0; kk < total_stages; ++kk) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          uint8_t* sA = tiles + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          const uint32_t fb = full0 + 8u * (uint32_t)stage;
          if (kk < p.k_stages) {
            uint8_t* sSFA = sf + stage * C::SF_STAGE_BYTES;
            uint8_t* sSFB = sSFA + C::SFA_BYTES;
            if (even) tc::mbar_expect_tx(&full[stage], C::PAIR_TX);
            tc::tma_load_2d_pair(sA, &mapA, fb, kk * 128, arow);
            tc::tma_load_2d_pair(sB, &mapB, fb, kk * 128, brow);
            // scale tiles: 512-byte atoms, 4 per stage and 128-row block; 8-byte elements
            tc::tma_load_1d_pair(sSFA, &mapSa, fb, (int32_t)(((int64_t)(arow / 128) * p.kb_tiles + kk * 4) * 64));
#pragma unroll
            for (int a = 0; a < 2; ++a)
              tc::tma_load_1d_pair(sSFB + a * 2048, &mapSb, fb,
                                   (int32_t)(((int64_t)(nb * 2 + a) * p.kb_tiles + kk * 4) * 64));
          } else {
            const int f = kk - p.k_stages;
            if (even) tc::mbar_expect_tx(&full[stage], C::PAIR_FOLD_TX);
            tc::tma_load_2d_pair(sA, &mapFa, fb, f * 64, arow);
            tc::tma_load_2d_pair(sB, &mapFb, fb, f * 64, brow);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && even) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t id_fp4 = tc::idesc_nvf4(C::BN, 256);
      const uint32_t id_bf16 = tc::idesc_bf16(C::BN, 256);
      for (int tile = pair; tile < num_tiles && !*abort_flag; tile += npairs, ++it) {
        if (!tc::mbar_wait(tmem_empty, ((uint32_t)it & 1u) ^ 1u, abort_flag)) {
          *abort_flag = 1;
          raise_status(p.status, METIS_DEV_TIMEOUT);
          break;
        }
        tc::tc_fence_after();
        for (int kk = 0; kk < total_stages; ++kk) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag) ||
              !tc::mbar_wait(&sf_ready[stage], phase, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          tc::tc_fence_after();
          const uint8_t* sA = tiles + stage * C::STAGE_BYTES;
          const uint8_t* sB = sA + C::A_BYTES;
          const uint64_t adesc = tc::sdesc_sw128(tc::smem_addr(sA));
          const uint64_t bdesc = tc::sdesc_sw128(tc::smem_addr(sB));
          if (kk < p.k_stages) {
            const uint32_t t_sfa = tmem + C::ACC_COLS + stage * C::SF_SET_COLS;
            const uint32_t t_sfb = t_sfa + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc::mma_nvf4_pair(tmem, adesc + 2 * j, bdesc + 2 * j, id_fp4, t_sfa + 4 * j,
                                t_sfb + C::SFB_COLS_PER_K * j, (kk || j) ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc::mma_bf16_pair(tmem, adesc + 2 * j, bdesc + 2 * j, id_bf16, (kk || j) ? 1u : 0u);
          }
          tc::tc_commit_pair(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (*abort_flag) break;
        tc::tc_commit_pair(tmem_full, 0x3);
      }
      // let every issued tensor-core operation finish before the memory is released
      tc::tc_commit_pair(drain, 0x1);
      tc::mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ scale copies (even CTA)
    // Warp 10 copies SFA of k-steps 0-1 and the first 128-row atom of SFB, warp 11 SFA
    // of k-steps 2-3 and the second atom: six pair-wide copies each per stage.
    const int part = warp - 10;
    if (lane == 0 && even) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < num_tiles && !*abort_flag; tile += npairs) {
        for (int kk = 0; kk < total_stages; ++kk) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            raise_status(p.status, METIS_DEV_TIMEOUT);
            break;
          }
          tc::tc_fence_after();
          if (kk < p.k_stages) {
            const uint8_t* sSFA = sf + stage * C::SF_STAGE_BYTES;
            const uint8_t* sSFB = sSFA + C::SFA_BYTES;
            const uint32_t t_sfa = tmem + C::ACC_COLS + stage * C::SF_SET_COLS;
            const uint32_t t_sfb = t_sfa + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if ((j >> 1) == part)
                tc::tc_copy_32x128b_x4_pair(t_sfa + 4 * j, tc::sdesc_scales(tc::smem_addr(sSFA + 512 * j)));
              tc::tc_copy_32x128b_x4_pair(t_sfb + C::SFB_COLS_PER_K * j + 4 * part,
                                          tc::sdesc_scales(tc::smem_addr(sSFB + 2048 * part + 512 * j)));
            }
          }
          tc::tc_commit_pair(&sf_ready[stage], 0x1);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // The accumulator is loaded into registers and released at once; the scaled tile
    // goes through the warp's shared-memory boxes (128-byte swizzle, so the row-per-lane
    // writes are conflict-free) and leaves by TMA stores, which the warp does not wait
    // for until it reuses the boxes one tile later.
    const int q = warp & 3;                 // tensor-memory lane quarter of this warp
    const int h = (warp - 2) >> 2;          // column half
    constexpr int kColsPerWarp = C::BN / 2;
    const float alpha = (p.ga ? *p.ga : 1.0f) * (p.gb ? *p.gb : 1.0f) * p.alpha_extra;
    const uint32_t empty_bar = tc::cluster_addr(tmem_empty, 0);
    uint8_t* box = epi + (warp - 2) * C::EPI_WARP_BYTES;
    const bool f32 = p.c_dtype == METIS_OUT_F32;
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tmem_full, (uint32_t)it & 1u, abort_flag));
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          raise_status(p.status, METIS_DEV_TIMEOUT);
        }
        break;
      }
      tc::tc_fence_after();
      const int mb = tile % p.m_tiles;
      const int nb = tile / p.m_tiles;
      const int col0 = h * kColsPerWarp;
      float v[kColsPerWarp];
#pragma unroll
      for (int c = 0; c < kColsPerWarp; c += 32) {
        float t[32];
        tc::tmem_load_32cols(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(col0 + c), t);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[c + i] = t[i];
      }
      tc::tmem_load_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster(empty_bar);

      const int32_t y = mb * 256 + (int)rank * 128 + q * 32;
      const int32_t x0 = nb * C::BN + col0;
      // 16-byte chunk j of a 128-byte box row r sits at position j ^ (r mod 8)
      const int swz = lane & 7;
      // one box of 128 bytes per row at a time: 64 bf16 or 32 fp32 columns
      constexpr int kBoxCols16 = 64, kBoxCols32 = 32;
      if (!f32) {
#pragma unroll
        for (int bx = 0; bx < kColsPerWarp / kBoxCols16; ++bx) {
          if (lane == 0) tc::bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {        // 8 bf16 columns per 16-byte chunk
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int col = kBoxCols16 * bx + 8 * c + 2 * i;
              const float a = v[col] * alpha * (p.col_scale ? p.col_scale[x0 + col] : 1.0f);
              const float b = v[col + 1] * alpha * (p.col_scale ? p.col_scale[x0 + col + 1] : 1.0f);
              const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
              w[i] = *reinterpret_cast<const uint32_t*>(&pr);
            }
            *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ swz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_2d(&mapC, box, x0 + kBoxCols16 * bx, y);
            tc::bulk_commit_group();
          }
        }
      } else {
#pragma unroll
        for (int bx = 0; bx < kColsPerWarp / kBoxCols32; ++bx) {
          if (lane == 0) tc::bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {        // 4 fp32 columns per 16-byte chunk
            const int col = kBoxCols32 * bx + 4 * c;
            float o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o[i] = v[col + i] * alpha * (p.col_scale ? p.col_scale[x0 + col + i] : 1.0f);
            *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ swz) << 4)) =
                make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                           __float_as_uint(o[3]));
          }
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_2d(&mapC, box, x0 + kBoxCols32 * bx, y);
            tc::bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) tc::bulk_wait_all();   // stores complete before the boxes go away
    __syncwarp();
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();   // no cross-CTA access is outstanding past this point
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  return enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 1-D map over a scale buffer viewed as 8-byte elements, 2 KB boxes (four 512-byte
// scale atoms); the buffer start is 16-byte aligned and every box starts on a 2 KB multiple.
bool make_map_1d_u64(CUtensorMap* map, const void* base, uint64_t bytes) {
  const cuuint64_t dims[1] = {bytes / 8};
  const cuuint64_t strides[1] = {bytes};   // unused for one dimension
  const cuuint32_t box[1] = {256};
  const cuuint32_t estr[1] = {1};
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 1, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
metis_status launch_spec(metis_ctx* ctx, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mFa,
                         const CUtensorMap& mFb, Params prm, double flops, bool profiled,
                         const CUtensorMap* extra_maps = nullptr) {
  using C = Cfg<BN>;
  auto kern = gemm_nvfp4_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(gemm)");
  int units = prm.m_tiles * prm.n_tiles * prm.k_splits;
  for (int e = 0; e < prm.n_extra; ++e) units += prm.extra[e].m_tiles * prm.extra[e].k_splits;
  const int grid = std::min(units, ctx->sm_count);
  // extra_maps: A1, B1, A2, B2 of a grouped launch (unused slots repeat the first problem's)
  const CUtensorMap& mA1 = extra_maps ? extra_maps[0] : mA;
  const CUtensorMap& mB1 = extra_maps ? extra_maps[1] : mB;
  const CUtensorMap& mA2 = extra_maps ? extra_maps[2] : mA;
  const CUtensorMap& mB2 = extra_maps ? extra_maps[3] : mB;
  const bool prof = ctx->profiling && profiled;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  if (prof) {
    cudaEventCreate(&ev0);
    cudaEventCreate(&ev1);
    cudaEventRecord(ev0, ctx->stream);
  }
  kern<<<grid, kThreads, C::SMEM, ctx->stream>>>(mA, mB, mFa, mFb, mA1, mB1, mA2, mB2, prm); count_launch();
  if (prof) {
    cudaEventRecord(ev1, ctx->stream);
    profile_record(ctx, kProfGemm, ev0, ev1, flops);
  }
  return check_cuda(ctx, cudaGetLastError(), "gemm launch");
}

template <int BN>
metis_status launch_bn(metis_ctx* ctx, const GemmArgs& a) {
  const int64_t p_rows = a.A->outer;
  const int64_t K = a.A->inner;
  const int64_t q_cols = a.q_cols;
  CUtensorMap mA, mB, mFa, mFb;
  if (!make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.A->codes, K / 2, p_rows, K / 2, 128, 128) ||
      !make_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.B->codes, K / 2, a.B->outer, K / 2, 128, BN))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the NVFP4 operands");
  if (a.fold_k > 0) {
    if (!make_map_2d(&mFa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Fa, a.fold_k, p_rows, (uint64_t)a.fold_k * 2, 64,
                     128) ||
        !make_map_2d(&mFb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Fb, a.fold_k, a.B->outer, (uint64_t)a.fold_k * 2,
                     64, BN))
      return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the fold operands");
  } else {
    mFa = mA;
    mFb = mB;
  }
  Params prm{};
  prm.sfa = a.A->scales;
  prm.sfb = a.B->scales;
  prm.kb_tiles = K / 64;
  prm.ga = a.A->tensor_scale;
  prm.gb = a.B->tensor_scale;
  prm.alpha_extra = a.alpha_extra;
  prm.col_scale = a.col_scale;
  prm.C = a.C;
  prm.ldc = a.ldc;
  prm.c_dtype = a.c_dtype;
  prm.m_tiles = (int)(p_rows / 128);
  prm.n_tiles = (int)(q_cols / BN);
  prm.k_stages = (int)(K / 256);
  prm.fold_stages = a.fold_k / 64;
  prm.k_splits = 1;
  prm.split_stride = 0;
  if (a.k_splits > 1) {
    if (a.c_dtype != METIS_OUT_F32) return fail(ctx, METIS_ERR_ARG, "split-K partials are fp32");
    const int total = prm.k_stages + prm.fold_stages;
    const int per = (total + a.k_splits - 1) / a.k_splits;
    prm.k_splits = (total + per - 1) / per;
    prm.split_stride = a.split_stride;
  }
  prm.status = ctx->status;
  return launch_spec<BN>(ctx, mA, mB, mFa, mFb, prm, 2.0 * (double)p_rows * (double)q_cols * (double)K,
                         q_cols >= 256);
}

// Both output dimensions multiples of 256, K a multiple of 256, one split.
metis_status launch_pair(metis_ctx* ctx, const GemmArgs& a) {
  using C = PairCfg;
  const int64_t p_rows = a.A->outer;
  const int64_t K = a.A->inner;
  const int64_t q_cols = a.q_cols;
  const int64_t kb_tiles = K / 64;
  CUtensorMap mA, mB, mFa, mFb, mSa, mSb;
  if (!make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.A->codes, K / 2, p_rows, K / 2, 128, 128) ||
      !make_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.B->codes, K / 2, a.B->outer, K / 2, 128, 128) ||
      !make_map_1d_u64(&mSa, a.A->scales, (uint64_t)(p_rows / 128) * kb_tiles * 512) ||
      !make_map_1d_u64(&mSb, a.B->scales, (uint64_t)((a.B->outer + 127) / 128) * kb_tiles * 512))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the NVFP4 operands");
  if (a.fold_k > 0) {
    if (!make_map_2d(&mFa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Fa, a.fold_k, p_rows, (uint64_t)a.fold_k * 2, 64,
                     128) ||
        !make_map_2d(&mFb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Fb, a.fold_k, a.B->outer, (uint64_t)a.fold_k * 2,
                     64, 128))
      return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the fold operands");
  } else {
    mFa = mA;
    mFb = mB;
  }
  CUtensorMap mC;
  const bool f32 = a.c_dtype == METIS_OUT_F32;
  if (!make_map_2d(&mC, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.C, q_cols,
                   p_rows, (uint64_t)a.ldc * (f32 ? 4 : 2), f32 ? 32 : 64, 32))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the output");
  Params prm{};
  prm.sfa = a.A->scales;
  prm.sfb = a.B->scales;
  prm.kb_tiles = kb_tiles;
  prm.ga = a.A->tensor_scale;
  prm.gb = a.B->tensor_scale;
  prm.alpha_extra = a.alpha_extra;
  prm.col_scale = a.col_scale;
  prm.C = a.C;
  prm.ldc = a.ldc;
  prm.c_dtype = a.c_dtype;
  prm.m_tiles = (int)(p_rows / 256);
  prm.n_tiles = (int)(q_cols / C::BN);
  prm.k_stages = (int)(K / 256);
  prm.fold_stages = a.fold_k / 64;
  prm.k_splits = 1;
  prm.split_stride = 0;
  prm.status = ctx->status;
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::SMEM);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(gemm pair)");
  const int tiles = prm.m_tiles * prm.n_tiles;
  const int grid = 2 * std::min(tiles, ctx->sm_count / 2);
  const bool prof = ctx->profiling;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  if (prof) {
    cudaEventCreate(&ev0);
    cudaEventCreate(&ev1);
    cudaEventRecord(ev0, ctx->stream);
  }
  gemm_nvfp4_pair_kernel<<<grid, kThreads, C::SMEM, ctx->stream>>>(mA, mB, mFa, mFb, mSa, mSb, mC, prm);
  count_launch();
  if (prof) {
    cudaEventRecord(ev1, ctx->stream);
    profile_record(ctx, kProfGemm, ev0, ev1, 2.0 * (double)p_rows * (double)q_cols * (double)K);
  }
  return check_cuda(ctx, cudaGetLastError(), "gemm pair launch");
}

template <int BN>
metis_status launch_bf16_bn(metis_ctx* ctx, const void* A, int64_t lda, int64_t rows, const void* B, int64_t ldb,
                            int64_t K, float* C, int64_t ldc, int splits) {
  CUtensorMap mFa, mFb;
  if (!make_map_2d(&mFa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, rows, (uint64_t)lda * 2, 64, 128) ||
      !make_map_2d(&mFb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, BN, (uint64_t)ldb * 2, 64, BN))
    return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the bf16 operands");
  Params prm{};
  prm.kb_tiles = 0;
  prm.alpha_extra = 1.0f;
  prm.C = C;
  prm.ldc = ldc;
  prm.c_dtype = METIS_OUT_F32;
  prm.m_tiles = (int)(rows / 128);
  prm.n_tiles = 1;
  prm.k_stages = 0;
  prm.fold_stages = (int)(K / 64);
  prm.k_splits = normalize_splits(K, splits);  // no empty split
  prm.split_stride = rows * ldc;
  prm.status = ctx->status;
  return launch_spec<BN>(ctx, mFa, mFb, mFa, mFb, prm, 2.0 * (double)rows * BN * (double)K, false);
}

// Up to three thin NVFP4 GeMMs (the same column width BN and contraction length, fp32
// outputs, no fold) in one persistent launch: the CTAs take the problems' work units in
// order, so the problems share the SMs without a launch between them.
template <int BN>
metis_status launch_group_bn(metis_ctx* ctx, const GemmArgs* g, int n) {
  const int64_t K = g[0].A->inner;
  CUtensorMap maps[6];
  for (int i = 0; i < n; ++i) {
    if (!make_map_2d(&maps[2 * i], CU_TENSOR_MAP_DATA_TYPE_UINT8, g[i].A->codes, K / 2, g[i].A->outer, K / 2, 128,
                     128) ||
        !make_map_2d(&maps[2 * i + 1], CU_TENSOR_MAP_DATA_TYPE_UINT8, g[i].B->codes, K / 2, g[i].B->outer, K / 2,
                     128, BN))
      return fail(ctx, METIS_ERR_CUDA, "cuTensorMapEncodeTiled failed for a grouped GeMM operand");
  }
  for (int i = n; i < 3; ++i) maps[2 * i] = maps[0], maps[2 * i + 1] = maps[1];
  const int stages = (int)(K / 256);
  auto splits_of = [&](const GemmArgs& a) {
    const int per = (stages + std::max(a.k_splits, 1) - 1) / std::max(a.k_splits, 1);
    return (stages + per - 1) / per;
  };
  Params prm{};
  prm.sfa = g[0].A->scales;
  prm.sfb = g[0].B->scales;
  prm.kb_tiles = K / 64;
  prm.ga = g[0].A->tensor_scale;
  prm.gb = g[0].B->tensor_scale;
  prm.alpha_extra = 1.0f;
  prm.C = g[0].C;
  prm.ldc = g[0].ldc;
  prm.c_dtype = METIS_OUT_F32;
  prm.m_tiles = (int)(g[0].A->outer / 128);
  prm.n_tiles = 1;
  prm.k_stages = stages;
  prm.fold_stages = 0;
  prm.k_splits = splits_of(g[0]);
  prm.split_stride = g[0].split_stride;
  prm.status = ctx->status;
  prm.n_extra = n - 1;
  for (int i = 1; i < n; ++i) {
    Params::Extra& x = prm.extra[i - 1];
    x.sfa = g[i].A->scales;
    x.sfb = g[i].B->scales;
    x.ga = g[i].A->tensor_scale;
    x.gb = g[i].B->tensor_scale;
    x.C = static_cast<float*>(g[i].C);
    x.ldc = g[i].ldc;
    x.m_tiles = (int)(g[i].A->outer / 128);
    x.k_splits = splits_of(g[i]);
    x.split_stride = g[i].split_stride;
  }
  return launch_spec<BN>(ctx, maps[0], maps[1], maps[0], maps[1], prm, 0.0, false, maps + 2);
}

}  // namespace

namespace {
// Split-K count for `tiles` output tiles of `stages` K stages each on a persistent grid of
// sm_count CTAs: the one that minimizes rounds x (stages per unit + 3) + splits x
// split_cost, rounds = ceil(tiles x splits / sm_count) -- the last round of equal units
// otherwise leaves SMs idle (64 tiles in 5 splits: 320 units, 3 rounds, 72% busy) -- 3
// stage-times stand for a unit's pipeline fill and its partial-tile store, and split_cost
// (in stage-times) for writing and summing one more set of fp32 partials.  At most 16.
int wave_splits(metis_ctx* ctx, int64_t tiles, int stages, double split_cost = 0.0) {
  const int64_t sms = std::max(1, ctx->sm_count);
  int best = 1;
  double best_cost = -1;
  for (int s = 1; s <= std::min(16, stages); ++s) {
    const int per = (stages + s - 1) / s;
    const int eff = (stages + per - 1) / per;
    const int64_t rounds = (tiles * eff + sms - 1) / sms;
    const double cost = (double)(rounds * (per + 3)) + split_cost * eff;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = eff;
    }
  }
  return best;
}
}  // namespace

// NVFP4 GeMMs: K / 256 stages per 128-row tile.  bf16 GeMMs of width n: K / 64 stages per
// 128-row tile; a split's partials (rows x n fp32, written and read once) cost
// 8 rows n / (sm_count x the stage's 128 x 64 + n x 64 bf16 bytes) stage-times.
int fp4_splits(metis_ctx* ctx, int64_t tiles, int stages) { return wave_splits(ctx, tiles, stages); }
int bf16_splits(metis_ctx* ctx, int64_t rows, int64_t K, int n) {
  const double stage_bytes = 128.0 * 64 * 2 + (double)n * 64 * 2;
  const double split_cost = 8.0 * (double)rows * n / ((double)std::max(1, ctx->sm_count) * stage_bytes);
  return wave_splits(ctx, rows / 128, (int)(K / 64), split_cost);
}

metis_status launch_gemm_bf16(metis_ctx* ctx, const void* A, int64_t lda, int64_t rows, const void* B, int64_t ldb,
                              int n, int64_t K, float* C, int64_t ldc, int splits) {
  if (rows % 128 || K % 64 || lda % 8 || ldb % 8)
    return fail(ctx, METIS_ERR_SHAPE, "bf16 GeMM needs rows % 128, K % 64 and 16-byte row strides");
  if (splits < 1) splits = bf16_splits(ctx, rows, K, n);
  if (splits > 1 && (int64_t)splits * rows * ldc > (int64_t(1) << 40))
    return fail(ctx, METIS_ERR_SHAPE, "split output too large");
  switch (n) {
    case 32: return launch_bf16_bn<32>(ctx, A, lda, rows, B, ldb, K, C, ldc, splits);
    case 64: return launch_bf16_bn<64>(ctx, A, lda, rows, B, ldb, K, C, ldc, splits);
    case 128: return launch_bf16_bn<128>(ctx, A, lda, rows, B, ldb, K, C, ldc, splits);
    case 256: return launch_bf16_bn<256>(ctx, A, lda, rows, B, ldb, K, C, ldc, splits);
    default: return fail(ctx, METIS_ERR_SHAPE, "bf16 GeMM width must be 32, 64, 128 or 256");
  }
}

metis_status launch_gemm_nvfp4_group(metis_ctx* ctx, const GemmArgs* g, int n) {
  if (n < 1 || n > 3) return fail(ctx, METIS_ERR_ARG, "a grouped GeMM takes 1 to 3 problems");
  for (int i = 0; i < n; ++i) {
    if (g[i].q_cols != g[0].q_cols || g[i].A->inner != g[0].A->inner || g[i].fold_k != 0 ||
        g[i].c_dtype != METIS_OUT_F32 || g[i].col_scale || g[i].B->outer != 128 || g[i].A->outer % 128 ||
        g[i].A->inner % 256)
      return fail(ctx, METIS_ERR_SHAPE, "grouped GeMMs need one thin width, one K, fp32 outputs and no fold");
  }
  switch (g[0].q_cols) {
    case 16: return launch_group_bn<16>(ctx, g, n);
    case 32: return launch_group_bn<32>(ctx, g, n);
    case 64: return launch_group_bn<64>(ctx, g, n);
    default: return fail(ctx, METIS_ERR_SHAPE, "grouped GeMM width must be 16, 32 or 64");
  }
}

metis_status launch_gemm_nvfp4(metis_ctx* ctx, const GemmArgs& a) {
  // CTA pairs whenever both output dimensions are multiples of 256 (the layer's GeMMs)
  // (the output leaves by TMA stores: 16-byte aligned base and row pitch)
  const int64_t out_bytes = a.c_dtype == METIS_OUT_F32 ? 4 : 2;
  if (a.q_cols % 256 == 0 && a.A->outer % 256 == 0 && a.k_splits <= 1 && ctx->sm_count >= 2 &&
      reinterpret_cast<uintptr_t>(a.C) % 16 == 0 && (a.ldc * out_bytes) % 16 == 0)
    return launch_pair(ctx, a);
  if (a.q_cols % 256 == 0) return launch_bn<256>(ctx, a);
  if (a.q_cols == 128) return launch_bn<128>(ctx, a);
  if (a.q_cols == 64) return launch_bn<64>(ctx, a);
  if (a.q_cols == 32) return launch_bn<32>(ctx, a);
  if (a.q_cols == 16) return launch_bn<16>(ctx, a);
  return fail(ctx, METIS_ERR_SHAPE, "GeMM output columns must be a multiple of 256 or one of 16, 32, 64");
}

}  // namespace metis
