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
                                            float g_in, const uint32_t* amax_bits, int rounding, uint64_t seed, uint32_t tag, uint32_t step,
                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                            float* tensor_scale, uint32_t* status) {
  const int64_t nblk_row = cols / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const float g = amax_bits ? auto_tensor_scale(*amax_bits) : g_in;
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
                                            float g_in, const uint32_t* amax_bits, int rounding, uint64_t seed, uint32_t tag, uint32_t step,
                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                            float* tensor_scale, uint32_t* status) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const float g = amax_bits ? auto_tensor_scale(*amax_bits) : g_in;
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

// Maximum |x| over the finite entries, as fp32 bits (non-negative floats order like
// their bit patterns), one atomicMax per warp.  A warp walks whole rows in 16-byte
// vectors: 8 bf16 or 4 fp32 elements.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const __nv_bfloat16* __restrict__ M, int64_t rows,
                                                        int64_t cols, int64_t ld, uint32_t* amax_bits) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t cv = cols / 8;
  uint32_t best = 0;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint4* row = reinterpret_cast<const uint4*>(M + r * ld);
    for (int64_t c = lane; c < cv; c += 32) {
      const uint4 v = row[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a = (w[i] >> (16 * h)) & 0x7FFFu;
          if ((a & 0x7F80u) != 0x7F80u) best = max(best, a << 16);
        }
      }
    }
  }
  best = __reduce_max_sync(0xffffffffu, best);
  if (lane == 0 && best) atomicMax(amax_bits, best);
}

__global__ void __launch_bounds__(256) amax_f32_kernel(const float* __restrict__ R, int64_t rows, int64_t cols,
                                                       int64_t ld, uint32_t* amax_bits) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t cv = cols / 4;
  uint32_t best = 0;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint4* row = reinterpret_cast<const uint4*>(R + r * ld);
    for (int64_t c = lane; c < cv; c += 32) {
      const uint4 v = row[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t a = w[i] & 0x7FFFFFFFu;
        if ((a & 0x7F800000u) != 0x7F800000u) best = max(best, a);
      }
    }
  }
  best = __reduce_max_sync(0xffffffffu, best);
  if (lane == 0 && best) atomicMax(amax_bits, best);
}

// Decode of one NVFP4 tensor: a thread per 16-element block reads 8 code bytes and its
// scale byte (tile layout) and writes 16 fp32 values.  e2m1 x e4m3 x g is exact in fp32.
__global__ void __launch_bounds__(256) dequantize_nvfp4_kernel(const uint8_t* __restrict__ codes,
                                                               const uint8_t* __restrict__ scales,
                                                               const float* __restrict__ g_ptr, int64_t outer,
                                                               int64_t inner, float* __restrict__ out, int64_t ld) {
  const int64_t nb = inner / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= outer * nb) return;
  const int64_t o = idx / nb;
  const int64_t b = idx - o * nb;
  const float g = *g_ptr;
  const uint32_t sc =
      scales[((o >> 7) * (inner / 64) + (b >> 2)) * 512 + (o & 31) * 16 + ((o & 127) >> 5) * 4 + (b & 3)];
  const float s = e4m3_value(sc & 0x7Fu) * g;
  const uint2 packed = *reinterpret_cast<const uint2*>(codes + o * (inner / 2) + b * 8);
  const uint32_t w[2] = {packed.x, packed.y};
  // E2M1 magnitudes of codes 0..7; bit 3 is the sign
  const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  float* dst = out + o * ld + b * 16;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t c = (w[h] >> (4 * i)) & 0xFu;
      const float m = mag[c & 7u] * s;
      v[i] = (c & 8u) ? -m : m;
    }
    reinterpret_cast<float4*>(dst + 8 * h)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst + 8 * h)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

}  // namespace

cudaError_t launch_dequantize(const metis_nvfp4* t, float* out, int64_t ld, cudaStream_t st) {
  const int64_t n = t->outer * (t->inner / 16);
  dequantize_nvfp4_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(t->codes, t->scales, t->tensor_scale,
                                                                       t->outer, t->inner, out, ld);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_amax(const void* M, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax_bits,
                        int sm_count, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int64_t want = (rows + 7) / 8;   // 8 warps per block, one row per warp per pass
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, 4 * (int64_t)sm_count));
  if (bf16)
    amax_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(M), rows, cols, ld, amax_bits);
  else
    amax_f32_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(M), rows, cols, ld, amax_bits);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quantize_f32(const float* R, int64_t rows, int64_t cols, int64_t ld,
                                const metis_quant_params& q, const uint32_t* amax_bits, const metis_nvfp4* rowwise,
                                const metis_nvfp4* colwise, uint32_t* status, cudaStream_t st) {
  const int threads = 256;
  if (rowwise) {
    const int64_t n = rows * (cols / 16);
    quantize_rowwise_f32_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
        R, rows, cols, ld, q.tensor_scale, amax_bits, q.rounding, q.seed,
        stream_tag(q.operand_id, kPurposeSR, kSrRowwise),
        q.step, rowwise->codes, rowwise->scales, rowwise->tensor_scale, status); count_launch();
  }
  if (colwise) {
    const int64_t n = (rows / 16) * cols;
    quantize_colwise_f32_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
        R, rows, cols, ld, q.tensor_scale, amax_bits, q.rounding, q.seed,
        stream_tag(q.operand_id, kPurposeSR, kSrColwise),
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
