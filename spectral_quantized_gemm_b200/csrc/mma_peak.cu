// NVFP4 tensor-core throughput microbenchmark: block-scaled tcgen05 MMAs with no memory
// traffic, to measure the FP4 MMA rate a kernel can reach on this GPU.
//
// Persistent clusters of two CTAs, one per SM pair, as in the fused GeMM's pair kernel:
// each CTA fills one 256-element K stage of A (its 128 rows) and B (its 128 of the 256
// rows) in shared memory with a fixed byte pattern and copies one set of block scales
// (E4M3 1.0) into tensor memory once; then the even CTA's MMA thread issues `iters`
// stages of four tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16
// (M = 256, N = 256, K = 64) into one accumulator and waits for them.  Useful flops:
// 2 * 256 * 256 * 256 per stage per pair.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace metis {
namespace {

constexpr int kPeakThreads = 128;
constexpr int kTileBytes = 128 * 128;          // 128 rows x 256 FP4 elements
constexpr int kScaleBytes = 4 * 512;           // 4 scale atoms (k-steps) of 128 rows

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPeakThreads, 1)
    mma_peak_kernel(int64_t iters, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kTileBytes;
  uint8_t* sS = smem + 2 * kTileBytes;                       // scales: SFA 4 atoms, SFB 2 x 4 atoms
  uint64_t* bars = reinterpret_cast<uint64_t*>(sS + 3 * kScaleBytes);
  uint64_t* done = bars;                                     // MMAs (or scale copies) finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool even = tc::cluster_rank() == 0;

  // operands: a fixed pattern of E2M1 codes, E4M3 scales of 1.0 (0x38)
  for (int i = threadIdx.x; i < 2 * kTileBytes / 4; i += kPeakThreads)
    reinterpret_cast<uint32_t*>(sA)[i] = 0x3A5C2B19u * (uint32_t)(i + 1);
  for (int i = threadIdx.x; i < 3 * kScaleBytes / 4; i += kPeakThreads)
    reinterpret_cast<uint32_t*>(sS)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  tc::fence_proxy_async();   // generic-proxy writes visible to the tensor core
  if (warp == 0) {
    tc::tmem_alloc_pair(tmem_slot, 512);
    tc::tmem_relinquish_pair();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0 && even) {
    const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 272;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tc::tc_copy_32x128b_x4_pair(t_sfa + 4 * j, tc::sdesc_scales(tc::smem_addr(sS + 512 * j)));
#pragma unroll
      for (int a = 0; a < 2; ++a)
        tc::tc_copy_32x128b_x4_pair(t_sfb + 8 * j + 4 * a,
                                    tc::sdesc_scales(tc::smem_addr(sS + kScaleBytes + 2048 * a + 512 * j)));
    }
    const uint64_t adesc = tc::sdesc_sw128(tc::smem_addr(sA));
    const uint64_t bdesc = tc::sdesc_sw128(tc::smem_addr(sB));
    const uint32_t id = tc::idesc_nvf4(256, 256);
    for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tc::mma_nvf4_pair(tmem, adesc + 2 * j, bdesc + 2 * j, id, t_sfa + 4 * j, t_sfb + 8 * j, (it || j) ? 1u : 0u);
    }
    tc::tc_commit_pair(done, 0x1);
    if (!tc::mbar_wait(done, 0, nullptr)) raise_status(status, METIS_DEV_TIMEOUT);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

metis_status launch_mma_peak(metis_ctx* ctx, int64_t iters, double* flops) {
  const size_t smem = 2 * kTileBytes + 3 * kScaleBytes + 1024 + 64;
  cudaError_t e = cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return check_cuda(ctx, e, "cudaFuncSetAttribute(mma peak)");
  const int pairs = ctx->sm_count / 2;
  mma_peak_kernel<<<2 * pairs, kPeakThreads, smem, ctx->stream>>>(iters, ctx->status);
  count_launch();
  *flops = 2.0 * 256.0 * 256.0 * 256.0 * (double)iters * (double)pairs;
  return check_cuda(ctx, cudaGetLastError(), "mma peak launch");
}

}  // namespace metis
