// Device helpers shared by the libmetis kernels: Philox4x32-10, the E2M1/E4M3
// conversions of the NVFP4 block quantizer, and the device status word.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/metis.h"

namespace metis {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11).  Counter (c0..c3), key
// (k0, k1); ten rounds, the key bumped by the Weyl constants between rounds.
// ---------------------------------------------------------------------------
struct Words4 {
  uint32_t w[4];
};

__device__ __forceinline__ Words4 philox10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                           uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  Words4 out;
  out.w[0] = c0;
  out.w[1] = c1;
  out.w[2] = c2;
  out.w[3] = c3;
  return out;
}

// Stream layout: key = seed, counter = (q lo, q hi, tag, step),
// tag = operand_id << 8 | purpose << 4 | sub.
enum : uint32_t { kPurposeSample = 1, kPurposeOmega = 2, kPurposeSR = 3 };
enum : uint32_t { kSrRowwise = 0, kSrColwise = 1, kSrLeft = 2, kSrRight = 3 };

__host__ __device__ __forceinline__ uint32_t stream_tag(uint32_t operand_id, uint32_t purpose,
                                                        uint32_t sub) {
  return ((operand_id & 0xFFFFFFu) << 8) | ((purpose & 0xFu) << 4) | (sub & 0xFu);
}

__device__ __forceinline__ Words4 stream_call(uint64_t seed, uint32_t tag, uint32_t step, uint64_t q) {
  return philox10((uint32_t)q, (uint32_t)(q >> 32), tag, step, (uint32_t)seed,
                  (uint32_t)(seed >> 32));
}

// ---------------------------------------------------------------------------
// Format conversions.  PTX cvt with .rn.satfinite: round to nearest even,
// saturating to the largest finite value; the packed destination takes the
// first source operand in its upper half.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_code_rn(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return (uint32_t)(r & 0xFFu);
}

// Exact fp32 value of a non-negative E4M3 code (OCP fn).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xFu;
  const uint32_t m = code & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9
  // (8 + m) * 2^(e - 10), built from the exponent bits
  const float p2 = __uint_as_float((e - 10u + 127u) << 23);
  return (float)(8u + m) * p2;
}

// Two fp32 values already on (or to be rounded to) the E2M1 grid -> one byte,
// `lo` in bits 0-3 and `hi` in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Stochastic rounding of four scaled values onto the E2M1 grid with 32 random bits w
// (codes of x0..x3 in bits 0-3 .. 12-15).  Per element, sign kept and |x| >= 6 giving 6:
// with lo <= |x| < hi the neighbouring magnitudes and p = (|x| - lo) / (hi - lo), the
// magnitude rounds up iff floor(p * 2^16) + F >= 2^16, where F is the element's 16-bit
// field of w: x0 takes bytes b2:b0, x1 the same 16 bits reversed, x2 takes b3:b1, x3
// those reversed.  The conversion instruction applies exactly this rule.
__device__ __forceinline__ uint32_t e2m1x4_sr(float x0, float x1, float x2, float x3, uint32_t w) {
  uint16_t r;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=h"(r) : "f"(x3), "f"(x2), "f"(x1), "f"(x0), "r"(w));
  return (uint32_t)r;
}

// Byte offset of the scale of (row o, block b) inside the tiled scale array of
// an NVFP4 tensor whose inner dimension has `kb_tiles` = inner/64 tiles.
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t o, int64_t b, int64_t kb_tiles) {
  return ((o >> 7) * kb_tiles + (b >> 2)) * 512 + (o & 31) * 16 + ((o & 127) >> 5) * 4 + (b & 3);
}

// ---------------------------------------------------------------------------
// NVFP4 block rule.  Given the block maximum and the tensor scale g, returns
// the E4M3 scale code and the fp32 reciprocal of the decode scale d = s*g.
// ---------------------------------------------------------------------------
struct BlockScale {
  uint32_t code;
  float rcp;  // 1 / (s * g), IEEE round-to-nearest; 0 for an all-zero block
};

__device__ __forceinline__ BlockScale block_scale(float amax, float g) {
  BlockScale bs;
  const float target = __fdiv_rn(amax, __fmul_rn(6.0f, g));
  uint32_t code = e4m3_code_rn(target);
  if (amax > 0.0f && code == 0) code = 1;  // smallest E4M3 value 2^-9
  bs.code = code;
  bs.rcp = code ? __frcp_rn(__fmul_rn(e4m3_value(code), g)) : 0.0f;
  return bs;
}

// Codes of one 16-element block whose values are already multiplied by the block's
// reciprocal scale, packed two per byte (element 2i in the low nibble of byte i).
// rounding 0: round to nearest even; 1: stochastic, with the four words of the Philox
// call of counter e0 / 16 (e0 = the block's first element index, a multiple of 16).
__device__ __forceinline__ uint2 encode_block16(const float (&x)[16], int rounding, uint64_t seed, uint32_t tag,
                                                uint32_t step, uint64_t e0) {
  uint2 r;
  if (rounding) {
    const Words4 w = stream_call(seed, tag, step, e0 >> 4);
    r.x = e2m1x4_sr(x[0], x[1], x[2], x[3], w.w[0]) | (e2m1x4_sr(x[4], x[5], x[6], x[7], w.w[1]) << 16);
    r.y = e2m1x4_sr(x[8], x[9], x[10], x[11], w.w[2]) | (e2m1x4_sr(x[12], x[13], x[14], x[15], w.w[3]) << 16);
  } else {
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = e2m1x2_rn(x[2 * i], x[2 * i + 1]);
    r.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    r.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  }
  return r;
}

// Decode tensor scale chosen from the data: the smallest power of two g with
// 2 * amax <= 6 * 448 * g, i.e. amax <= 1344 * g (amax = max |x| over the finite
// entries, given as fp32 bits); 1 for amax = 0; exponent clamped to [-126, 127].
// With amax = 1.m * 2^(E - 127) and 1344 = 1.3125 * 2^10: g = 2^(E - 137) when
// 1.m <= 1.3125 (mantissa field <= 0x280000), else 2^(E - 136).
__device__ __forceinline__ float auto_tensor_scale(uint32_t amax_bits) {
  if (amax_bits == 0) return 1.0f;
  const int E = (int)(amax_bits >> 23);
  if (E == 0) return __uint_as_float(1u << 23);                  // subnormal amax: 2^-126
  int e = ((amax_bits & 0x7FFFFFu) <= 0x280000u) ? E - 137 : E - 136;
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Tensor scale of a factor: g = pow2_ceil(max|F| / (6 * 448)), so that every block scale
// fits E4M3 and dequantized factors stay exact in bf16.
// Smallest power of two >= t (t >= 0 finite); 1 for t == 0.
__device__ __forceinline__ float pow2_ceil(float t) {
  if (!(t > 0.0f)) return 1.0f;
  const uint32_t bits = __float_as_uint(t);
  const uint32_t e = bits >> 23, m = bits & 0x7FFFFFu;
  if (e == 0) {  // subnormal: t = m * 2^-149
    const uint32_t top = 31u - __clz(m);
    const uint32_t p = (m & (m - 1)) ? top + 1 : top;
    return p >= 23 ? __uint_as_float(1u << 23) : __uint_as_float(1u << p);
  }
  if (m == 0) return t;
  return __uint_as_float((e + 1) << 23);
}

__device__ __forceinline__ void raise_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace metis
