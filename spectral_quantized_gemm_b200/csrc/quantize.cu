// NVFP4 block quantization kernels.
//
// Method: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
// background section (NVFP4: E2M1 values, 16-element blocks, one FP8 scale per
// block from the block maximum) and training strategy (W4A4G4, stochastic
// rounding on by default).  The block rule:
//   s = E4M3_RN(amax / (6 g)) (2^-9 if that rounds to 0 for a non-zero block),
//   x = v * RN(1 / (s g)),  code = E2M1_RN(x) or stochastic rounding of x.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "internal.h"

namespace metis {
namespace {

// One thread per 16-element block of the row-wise view (blocks along columns).
__global__ void quantize_rowwise_f32_kernel(const float* __restrict__ R, int64_t rows, int64_t cols, int64_t ld,
                                            float g, int rounding, uint64_t seed, uint32_t tag, uint32_t step,
                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                            float* tensor_scale, uint32_t* status) {
  const int64_t nblk_row = cols / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx == 0 && tensor_scale) *tensor_scale = g;
  if (idx >= rows * nblk_row) return;
  const int64_t o = idx / nblk_row;
  const int64_t b = idx - o * nblk_row;
  const float4* src = reinterpret_cast<const float4*>(R + o * ld + b * 16);
  float v[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 t = src[i];
    v[4 * i] = t.x;
    v[4 * i + 1] = t.y;
    v[4 * i + 2] = t.z;
    v[4 * i + 3] = t.w;
  }
  float amax = 0.0f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    finite &= isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  const BlockScale bs = block_scale(amax, g);
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __fmul_rn(v[i], bs.rcp);
  const uint64_t e0 = (uint64_t)o * (uint64_t)cols + (uint64_t)b * 16;
  uint2 packed = encode_block16(x, rounding, seed, tag, step, e0);
  if (bs.code == 0) packed = make_uint2(0, 0);
  *reinterpret_cast<uint2*>(codes + o * (cols / 2) + b * 8) = packed;
  scales[scale_offset(o, b, cols / 64)] = (uint8_t)bs.code;
}

// One thread per 16-row block of one column (column-wise view, blocks along rows).
// Consecutive threads take consecutive columns so the loads coalesce.
__global__ void quantize_colwise_f32_kernel(const float* __restrict__ R, int64_t rows, int64_t cols, int64_t ld,
                                            float g, int rounding, uint64_t seed, uint32_t tag, uint32_t step,
                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                            float* tensor_scale, uint32_t* status) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx == 0 && tensor_scale) *tensor_scale = g;
  const int64_t nblk = rows / 16;
  if (idx >= nblk * cols) return;
  const int64_t b = idx / cols;   // block along rows
  const int64_t j = idx - b * cols;  // column = outer index of the transposed view
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = R[(b * 16 + i) * ld + j];
  float amax = 0.0f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    finite &= isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  if (!finite) raise_status(status, METIS_DEV_NONFINITE);
  const BlockScale bs = block_scale(amax, g);
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __fmul_rn(v[i], bs.rcp);
  const uint64_t e0 = (uint64_t)j * (uint64_t)rows + (uint64_t)b * 16;
  uint2 packed = encode_block16(x, rounding, seed, tag, step, e0);
  if (bs.code == 0) packed = make_uint2(0, 0);
  *reinterpret_cast<uint2*>(codes + j * (rows / 2) + b * 8) = packed;
  scales[scale_offset(j, b, rows / 64)] = (uint8_t)bs.code;
}

// out = fp32(M - (U diag(S)) V^T), a 64 x 64 tile per block, 4 x 4 per thread.
__global__ void residual_f32_kernel(const __nv_bfloat16* __restrict__ M, int64_t rows, int64_t cols, int64_t ld,
                                    const float* __restrict__ U, const float* __restrict__ S,
                                    const float* __restrict__ V, int k, float* __restrict__ out) {
  __shared__ float us[64][65];
  __shared__ float vs[64][65];
  const int64_t r0 = (int64_t)blockIdx.y * 64;
  const int64_t c0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int t0 = 0; t0 < k; t0 += 64) {
    const int kt = min(64, k - t0);
    for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
      const int r = i / 64, t = i % 64;
      us[r][t] = t < kt ? U[(r0 + r) * k + t0 + t] * S[t0 + t] : 0.0f;
      vs[r][t] = t < kt ? V[(c0 + r) * k + t0 + t] : 0.0f;
    }
    __syncthreads();
    for (int t = 0; t < kt; ++t) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = us[ty * 4 + i][t];
        b[i] = vs[tx * 4 + i][t];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = c0 + tx * 4 + j;
      out[r * cols + c] = __bfloat162float(M[r * ld + c]) - acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_quantize_f32(const float* R, int64_t rows, int64_t cols, int64_t ld,
                                const metis_quant_params& q, const metis_nvfp4* rowwise,
                                const metis_nvfp4* colwise, uint32_t* status, cudaStream_t st) {
  const int threads = 256;
  if (rowwise) {
    const int64_t n = rows * (cols / 16);
    quantize_rowwise_f32_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
        R, rows, cols, ld, q.tensor_scale, q.rounding, q.seed, stream_tag(q.operand_id, kPurposeSR, kSrRowwise),
        q.step, rowwise->codes, rowwise->scales, rowwise->tensor_scale, status); count_launch();
  }
  if (colwise) {
    const int64_t n = (rows / 16) * cols;
    quantize_colwise_f32_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
        R, rows, cols, ld, q.tensor_scale, q.rounding, q.seed, stream_tag(q.operand_id, kPurposeSR, kSrColwise),
        q.step, colwise->codes, colwise->scales, colwise->tensor_scale, status); count_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_residual_f32(const void* M_bf16, int64_t rows, int64_t cols, int64_t ld, const float* U,
                                const float* S, const float* V, int32_t k, float* out, uint32_t* status,
                                cudaStream_t st) {
  (void)status;
  dim3 grid((unsigned)(cols / 64), (unsigned)(rows / 64));
  residual_f32_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(M_bf16), rows, cols, ld, U, S,
                                            V, k, out); count_launch();
  return cudaGetLastError();
}


}  // namespace metis
