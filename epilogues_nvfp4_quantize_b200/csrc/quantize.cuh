// nvfp4_quantize: bf16 -> NVFP4 (E2M1 codes, E4M3 block scales in the tensor-core scale
// layout, FP32 per-tensor scale). HBM-bound: an optional amax pass, then one pass that
// reads 128 bytes and writes 36 bytes per thread.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"

namespace nvfp4 {

// amax(|x|) over a rows x cols bf16 tensor, folded into *amax_bits (float bits, the
// caller zeroes it first) with one atomicMax per block. Each thread keeps four 16-byte
// loads in flight per iteration.
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ldx,
                                                   unsigned int* __restrict__ amax_bits) {
  const int64_t upr = cols >> 3;  // 16-byte units per row
  const int64_t total = rows * upr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u0 < total; u0 += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t u = u0 + i * stride;
      if (u < total) {
        const int64_t r = u / upr, c = u - r * upr;
        v[i] = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + c * 8));
      } else {
        v[i] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu, v[i].z & 0x7FFF7FFFu,
                             v[i].w & 0x7FFF7FFFu};
#pragma unroll
      for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(bf16_lo(w[k]), bf16_hi(w[k])));
    }
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

// Quantise rows x cols (cols % 64 == 0). One thread owns 64 adjacent values of a row:
// four 16-blocks, i.e. one 4-byte scale word and 32 bytes of codes. Threads cover rows
// padded to 128 so that the padding scale words are written as 0. With `interleave`,
// output row 2j reads input row j and output row 2j+1 reads input row rows/2 + j.
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
  const int64_t cpr = cols >> 6;  // 64-value groups per row
  const int64_t rows_pad = (rows + 127) & ~static_cast<int64_t>(127);
  const int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (u >= rows_pad * cpr) return;
  const int64_t r = u / cpr, c = u - r * cpr;
  uint32_t word = 0;
  if (r < rows) {
    const int64_t src = interleave ? ((r & 1) ? (rows >> 1) + (r >> 1) : (r >> 1)) : r;
    const uint4* p = reinterpret_cast<const uint4*>(x + src * ldx + c * 64);
    uint4 q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __ldg(p + i);
    uint32_t cw[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t w[8] = {q[2 * b].x, q[2 * b].y, q[2 * b].z, q[2 * b].w,
                             q[2 * b + 1].x, q[2 * b + 1].y, q[2 * b + 1].z, q[2 * b + 1].w};
      const uint32_t s = quant_block16_bf16(w, G, enc, cw[2 * b], cw[2 * b + 1]);
      word |= s << (8 * b);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + r * (cols >> 1) + c * 32);
    dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
  }
  *reinterpret_cast<uint32_t*>(sf + sf_word_offset(r, 4 * c, cols >> 4)) = word;
}

}  // namespace nvfp4
