// Stand-alone op kernels of the unfused comparison: the GEMM writes its bf16 output to
// HBM, then one of these reads it back, applies the op and writes again (the round trip
// that "Serving sub-second Ideogram v4 without quality loss", section "Epilogue fusion
// in brief", sets out to remove). Both are HBM-bound and fully coalesced.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"

namespace nvfp4 {

// One warp per (row, head): y = x * rsqrt(mean(x^2) + eps) * w[col] over head_dim columns.
template <int HD>
__global__ void __launch_bounds__(256) rmsnorm_heads_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            int64_t ldx, const float* __restrict__ w,
                                                            int64_t n_norm_cols, float eps,
                                                            uint16_t* __restrict__ y, int64_t ldy) {
  constexpr int PER = HD / 32;  // values per lane: 8 or 4
  const int64_t hpr = n_norm_cols / HD;
  const int64_t gw = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  if (gw >= rows * hpr) return;
  const int lane = threadIdx.x & 31;
  const int64_t r = gw / hpr, h = gw - r * hpr;
  const int64_t col = h * HD + lane * PER;
  float v[PER];
  if constexpr (PER == 8) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + col));
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(u[i]);
      v[2 * i + 1] = bf16_hi(u[i]);
    }
  } else {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(x + r * ldx + col));
    v[0] = bf16_lo(q.x);
    v[1] = bf16_hi(q.x);
    v[2] = bf16_lo(q.y);
    v[3] = bf16_hi(q.y);
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < PER; ++i) ss = fmaf(v[i], v[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = rsqrtf(ss * (1.0f / HD) + eps);
  uint32_t out[PER / 2];
#pragma unroll
  for (int i = 0; i < PER / 2; ++i) {
    const float2 wv = __ldg(reinterpret_cast<const float2*>(w + col + 2 * i));
    out[i] = pack_bf16x2(v[2 * i] * rstd * wv.x, v[2 * i + 1] * rstd * wv.y);
  }
  if constexpr (PER == 8) {
    *reinterpret_cast<uint4*>(y + r * ldy + col) = make_uint4(out[0], out[1], out[2], out[3]);
  } else {
    *reinterpret_cast<uint2*>(y + r * ldy + col) = make_uint2(out[0], out[1]);
  }
}

__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// One thread per 8 outputs: y[r, j] = silu(c[r, j]) * c[r, nh + j].
__global__ void __launch_bounds__(256) swiglu_kernel(const uint16_t* __restrict__ c, int64_t rows,
                                                     int64_t nh, int64_t ldc, uint16_t* __restrict__ y,
                                                     int64_t ldy) {
  const int64_t per_row = nh >> 3;
  const int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (u >= rows * per_row) return;
  const int64_t r = u / per_row, j = (u - r * per_row) * 8;
  const uint4 g = __ldg(reinterpret_cast<const uint4*>(c + r * ldc + j));
  const uint4 p = __ldg(reinterpret_cast<const uint4*>(c + r * ldc + nh + j));
  const uint32_t gg[4] = {g.x, g.y, g.z, g.w};
  const uint32_t pp[4] = {p.x, p.y, p.z, p.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[i] = pack_bf16x2(silu_f32(bf16_lo(gg[i])) * bf16_lo(pp[i]), silu_f32(bf16_hi(gg[i])) * bf16_hi(pp[i]));
  }
  *reinterpret_cast<uint4*>(y + r * ldy + j) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Bounded-wait self-test: wait on a barrier that nothing completes.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait(&bar, 0, &abort_flag, limit_ns, 100);
  }
  __syncthreads();
}

}  // namespace nvfp4
