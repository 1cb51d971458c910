// nvfp4_quantize: bf16 -> NVFP4 (E2M1 codes, E4M3 block scales in the tensor-core scale
// layout, FP32 per-tensor scale). HBM-bound; one thread owns 8 adjacent values, a lane
// pair owns one 16-block, and 8 lanes own the 4 blocks of one scale word.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"

namespace nvfp4 {

// amax(|x|) over a rows x cols bf16 tensor, folded into *amax_bits (float bits, the
// caller zeroes it first) with one atomicMax per block.
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ldx,
                                                   unsigned int* __restrict__ amax_bits) {
  const int64_t upr = cols >> 3;  // 16-byte units per row
  const int64_t total = rows * upr;
  float m = 0.0f;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = u / upr, c = u - r * upr;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + c * 8));
    const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu,
                           v.w & 0x7FFF7FFFu};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(bf16_lo(w[i]), bf16_hi(w[i])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) b = fmaxf(b, wmax[i]);
    if (b > 0.0f) atomicMax(amax_bits, __float_as_uint(b));
  }
}

// Quantise rows x cols (cols % 64 == 0). Threads cover rows padded to 128 so that the
// padding scale bytes are written as 0. With `interleave`, output row 2j reads input
// row j and output row 2j+1 reads input row rows/2 + j.
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                       int64_t cols, int64_t ldx, int interleave,
                                                       const unsigned int* __restrict__ amax_bits,
                                                       float* __restrict__ gscale,
                                                       uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ sf) {
  float G;
  if (amax_bits != nullptr) {
    G = __fdiv_rn(__uint_as_float(*amax_bits), kGlobalDiv);
    if (blockIdx.x == 0 && threadIdx.x == 0) *gscale = G;
  } else {
    G = *gscale;
  }
  const float enc = scale_encode_factor(G);
  const int64_t upr = cols >> 3;
  const int64_t rows_pad = (rows + 127) & ~static_cast<int64_t>(127);
  const int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (u >= rows_pad * upr) return;  // whole warps only: rows_pad * upr is a multiple of 32
  const int64_t r = u / upr, c = u - r * upr;
  const bool valid = r < rows;
  float v[8];
  if (valid) {
    const int64_t src = interleave ? ((r & 1) ? (rows >> 1) + (r >> 1) : (r >> 1)) : r;
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(x + src * ldx + c * 8));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  const uint32_t s = block_scale_code(amax, enc);
  if (valid) {
    const uint32_t cw = block_codes8(v, s, G);
    *reinterpret_cast<uint32_t*>(codes + r * (cols >> 1) + c * 4) = cw;
  }
  const int lane = threadIdx.x & 31;
  const int base = lane & ~7;
  const uint32_t s0 = __shfl_sync(0xffffffffu, s, base);
  const uint32_t s1 = __shfl_sync(0xffffffffu, s, base + 2);
  const uint32_t s2 = __shfl_sync(0xffffffffu, s, base + 4);
  const uint32_t s3 = __shfl_sync(0xffffffffu, s, base + 6);
  if ((lane & 7) == 0) {
    const int64_t kb = c >> 1;  // first 16-block of this 64-column group
    *reinterpret_cast<uint32_t*>(sf + sf_word_offset(r, kb, cols >> 4)) =
        s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

}  // namespace nvfp4
