// Device-side NVFP4 codec: E2M1 / E4M3 conversions and the 16-element block quantiser.
//
// The block rule (one unsigned E4M3 scale per 16 values, FP32 per-tensor scale G) is
// evaluated with exactly these IEEE float32 operations, in this order:
//   enc = rcp_rn(6 * G);  s = E4M3_rn_satfinite(min(amax_b * enc, 448))  (0 if amax_b == 0)
//   d = e4m3(s) * G;      q_i = E2M1_rn_satfinite(x_i * rcp_rn(d))        (0 if d == 0)
// FP4 is E2M1 as in "Serving sub-second Ideogram v4 without quality loss", section
// "Running the transformer in FP4"; static scales for inference follow its section
// "Quantization-aware distillation".
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace nvfp4 {

constexpr float kE4M3Max = 448.0f;
constexpr float kGlobalDiv = 2688.0f;  // 6 (largest E2M1) * 448 (largest E4M3)

// Eight floats -> four bytes of E2M1 codes; element 0 lands in bits 0-3.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// Non-negative float -> E4M3 code (round to nearest even, saturating).
__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// E4M3 code -> float (exact: every E4M3 value is a half).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

__device__ __forceinline__ float scale_encode_factor(float G) {
  return G > 0.0f ? __frcp_rn(__fmul_rn(6.0f, G)) : __int_as_float(0x7f800000);
}

// Scale code of a block whose largest magnitude is amax.
__device__ __forceinline__ uint32_t block_scale_code(float amax, float enc) {
  if (!(amax > 0.0f)) return 0u;
  return cvt_e4m3(fminf(__fmul_rn(amax, enc), kE4M3Max));
}

// Reciprocal of the decoded block scale d = e4m3(s) * G (0 when d is 0: the block's codes
// are then 0).
__device__ __forceinline__ float block_inv_scale(uint32_t s, float G) {
  const float d = __fmul_rn(e4m3_to_f32(s), G);
  return d > 0.0f ? __frcp_rn(d) : 0.0f;
}

// Codes of 8 values of a block, given the reciprocal r of its decoded scale.
__device__ __forceinline__ uint32_t block_codes8(const float* x, float r) {
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(x[i], r);
  return cvt_e2m1x8(y);
}

// Quantise one block of 16 values: returns the scale code, writes 8 bytes of codes.
__device__ __forceinline__ uint32_t quant_block16(const float* x, float G, float enc, uint32_t& c_lo,
                                                  uint32_t& c_hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t s = block_scale_code(amax, enc);
  const float r = block_inv_scale(s, G);
  c_lo = block_codes8(x, r);
  c_hi = block_codes8(x + 8, r);
  return s;
}

// Largest magnitude of 16 bf16 values packed in 8 words: max(|a|, |b|) per half with
// max.xorsign.abs (the sign it leaves is dropped at the end).
__device__ __forceinline__ float bf16x16_amax(const uint32_t* p) {
  uint32_t m = p[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(p[i]));
  return fmaxf(fabsf(__uint_as_float(m << 16)), fabsf(__uint_as_float(m & 0xFFFF0000u)));
}

// Quantise one block of 16 bf16 values packed in 8 words (bit-identical to quant_block16
// on the unpacked values).
__device__ __forceinline__ uint32_t quant_block16_bf16(const uint32_t* p, float G, float enc, uint32_t& c_lo,
                                                       uint32_t& c_hi) {
  const uint32_t s = block_scale_code(bf16x16_amax(p), enc);
  const float r = block_inv_scale(s, G);
  float x[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    x[2 * j] = __uint_as_float(p[j] << 16);
    x[2 * j + 1] = __uint_as_float(p[j] & 0xFFFF0000u);
  }
  c_lo = block_codes8(x, r);
  c_hi = block_codes8(x + 8, r);
  return s;
}

// Byte offset of the 4-byte scale word holding blocks kb..kb+3 (kb % 4 == 0) of `row`
// in the tensor-core scale layout (nkb = number of 16-blocks per row, a multiple of 4).
__device__ __forceinline__ int64_t sf_word_offset(int64_t row, int64_t kb, int64_t nkb) {
  const int64_t unit = (row >> 7) * (nkb >> 2) + (kb >> 2);
  const int r = static_cast<int>(row & 127);
  return unit * 512 + (r & 31) * 16 + (r >> 5) * 4;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<const uint32_t*>(&p);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 p = __floats2half2_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<const uint32_t*>(&p);
}

}  // namespace nvfp4
