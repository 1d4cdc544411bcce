// NVFP4 block quantization shared by the quantizer kernels and the scan's
// fused o quantization (one definition, so both produce the same bytes).
//
// Method: "Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the
// 'Fragile' Recurrence is Actually Robust" -- every 16-element block gets its
// own scale.  Two-level recipe, FP32 round-to-nearest one operation at a time:
// g_enc = 2688 / amax(tensor); per block s = E4M3_satfinite((amax_b / 6) g_enc),
// codes E2M1_satfinite(x (g_enc / s)), element 2j in the low nibble of byte j;
// scales in the tensor-core tiled layout (512-byte blocks of 128 rows x 4).
#pragma once
#include <float.h>
#include <stdint.h>

#include "common.cuh"

namespace gdn {
namespace {

// Input element types: bf16 (8 per 16-byte vector) or FP32 (4 per vector).
struct Bf16In {
  static constexpr int kPerVec = 8;
  __device__ static uint32_t absmax_bits(uint4 v) {  // FP32 bits of max |x|
    uint32_t m = 0;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m = max(m, w[i] & 0x7FFFu);
      m = max(m, (w[i] >> 16) & 0x7FFFu);
    }
    return m << 16;
  }
  __device__ static void to_f32(uint4 v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      out[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
  }
};
struct F32In {
  static constexpr int kPerVec = 4;
  __device__ static uint32_t absmax_bits(uint4 v) {
    return max(max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu), max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu));
  }
  __device__ static void to_f32(uint4 v, float* out) {
    out[0] = __uint_as_float(v.x);
    out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z);
    out[3] = __uint_as_float(v.w);
  }
};

__device__ __forceinline__ float encode_scale_from_amax(float amax) {
  if (amax == 0.0f) return 1.0f;
  float g = __fdiv_rn(2688.0f, amax);
  return (g > FLT_MAX) ? FLT_MAX : g;
}

// E4M3 byte -> FP32 value (exact).
__device__ __forceinline__ float e4m3_value(uint32_t s) {
  uint32_t e = (s >> 3) & 15u, m = s & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__device__ __forceinline__ uint32_t e4m3_satfinite(float v) {
  uint16_t out;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %1;\n\tmov.b16 %0, t;\n\t}"
      : "=h"(out)
      : "f"(v));
  return out & 0xFFu;
}

// Four pairs -> 4 bytes; element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float* r) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]));
  return out;
}

// Byte offset of the scale of (row R, 16-element group j) in the tiled layout.
__device__ __forceinline__ int64_t scale_offset(int64_t R, int64_t j, int64_t kc) {
  return (R >> 7) * kc * 512 + (j >> 2) * 512 + (R & 31) * 16 + ((R & 127) >> 5) * 4 + (j & 3);
}

// One 16-element block: E4M3 scale, eight packed code bytes, one scale byte.
template <typename In>
__device__ __forceinline__ void quant_block(const uint4 (&v)[16 / In::kPerVec], float g_enc, uint8_t* codes,
                                            uint8_t* scale) {
  constexpr int NV = 16 / In::kPerVec;
  uint32_t mb = 0;
#pragma unroll
  for (int i = 0; i < NV; ++i) mb = max(mb, In::absmax_bits(v[i]));
  const float amax_b = __uint_as_float(mb);
  const float s_f = __fmul_rn(__fdiv_rn(amax_b, 6.0f), g_enc);
  const uint32_t s = e4m3_satfinite(s_f);
  const float s_val = e4m3_value(s);
  uint2 packed = make_uint2(0u, 0u);
  if (s_val > 0.0f) {
    const float inv = __fdiv_rn(g_enc, s_val);
    float rr[16];
#pragma unroll
    for (int i = 0; i < NV; ++i) In::to_f32(v[i], rr + i * In::kPerVec);
#pragma unroll
    for (int i = 0; i < 16; ++i) rr[i] = __fmul_rn(rr[i], inv);
    packed.x = e2m1x8(rr);
    packed.y = e2m1x8(rr + 8);
  }
  *reinterpret_cast<uint2*>(codes) = packed;
  *scale = (uint8_t)s;
}

}  // namespace
}  // namespace gdn
