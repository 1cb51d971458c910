// nvfp4_quantize: bf16 -> NVFP4 (E2M1 codes, E4M3 block scales in the tensor-core scale
// layout, FP32 per-tensor scale). HBM-bound. amax_partial_kernel, then quantize_flat_kernel
// (contiguous x) or quantize_rows_kernel (other layouts), are the path of nvfp4_quantize and
// nvfp4_fake_quantize; quantize_kernel (one thread per 64
// values, plain loads) serves the allocation-free variant, whose amax reduction runs in
// kernels of its own.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"

namespace nvfp4 {

// Quantise rows x cols (cols % 64 == 0) with a per-tensor scale already derived (from
// *amax_bits, or *gscale when amax_bits is null). One thread owns 64 adjacent values of a row:
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

// Dequantised bf16 values of one 16-block: bf16(fp32(e2m1(q) * e4m3(s)) * G). The
// level-scale products are exact in f16 (at most 2 + 4 significant bits, magnitudes from
// 2^-10 to 2688), so they are formed two at a time with one f16x2 multiply.
__device__ __forceinline__ void dequant_block16_bf16(uint32_t c_lo, uint32_t c_hi, uint32_t s, float G,
                                                     uint32_t (&out)[8]) {
  uint32_t sv2;
  asm("{\n\t.reg .b16 h;\n\tcvt.rn.f16x2.e4m3x2 %0, %1;\n\tmov.b32 {h, _}, %0;\n\tmov.b32 %0, {h, h};\n\t}"
      : "=r"(sv2)
      : "h"(static_cast<uint16_t>(s & 0xFFu)));
  const uint32_t cw[2] = {c_lo, c_hi};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t lv2, p2;
      asm("{\n\t.reg .b8 c;\n\tcvt.u8.u32 c, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
          : "=r"(lv2)
          : "r"((cw[h] >> (8 * k)) & 0xFFu));
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p2) : "r"(lv2), "r"(sv2));
      const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(p2 & 0xFFFFu)));
      const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(p2 >> 16)));
      out[4 * h + k] = pack_bf16x2(__fmul_rn(lo, G), __fmul_rn(hi, G));
    }
  }
}

// =====================================================================================
// Two-kernel quantiser (the path of nvfp4_quantize and nvfp4_fake_quantize).
//
// 1. amax_partial_kernel streams x once (HBM-bound) and writes one partial max|x| per CTA
//    into the caller's workspace.
// 2. The quantise kernel is launched with programmatic dependent launch: its CTAs may
//    become resident while the first kernel drains, and wait (griddepcontrol.wait) until
//    that kernel's partials are visible. Each CTA reduces the partials to the tensor's amax,
//    derives G = amax / (6 * 448), and fills a shared table of the 127 block-scale
//    reciprocals 1 / (e4m3(s) * G). A lane quantises a 16-value block with one 32-byte
//    load, the block's E4M3 scale, one table lookup for the reciprocal, 16 products and 8
//    E2M1 conversions, and an 8-byte code store. quantize_flat_kernel gives each lane four
//    blocks of a 128-block warp task and builds the scale words with a byte transpose
//    within each quad; quantize_rows_kernel gives each lane one block of a 512-column row
//    chunk and builds them with two shuffles. Both walk x in the reverse order of the first
//    kernel's reads, so the data read last (likeliest still in L2) is quantised first.
// No grid barrier and no workspace clearing: every partial a call reads is written by the
// same call.
// =====================================================================================
namespace q2cfg {
constexpr int AMAX_THREADS = 512;
constexpr int QUANT_THREADS = 256;
constexpr int QUANT_WARPS = QUANT_THREADS / 32;
constexpr int MAX_PARTIALS = 1024;  // floats of workspace: one per CTA of the amax kernel
}  // namespace q2cfg

// 32 bytes (16 bf16) from global memory with an L2 eviction policy: one 256-bit access when
// the address is 32-byte aligned (V8), else two 128-bit accesses (16-byte aligned).
template <bool V8>
__device__ __forceinline__ void ld_global_32b(const void* p, uint64_t policy, uint32_t (&w)[8]) {
  if constexpr (V8) {
    asm("ld.global.nc.L2::cache_hint.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], %9;"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(p), "l"(policy));
  } else {
    const char* c = static_cast<const char*>(p);
    asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
        : "l"(c), "l"(policy));
    asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(c + 16), "l"(policy));
  }
}
template <bool V8>
__device__ __forceinline__ void st_global_32b(void* p, const uint32_t (&w)[8]) {
  if constexpr (V8) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
  } else {
    uint4* q = static_cast<uint4*>(p);
    q[0] = make_uint4(w[0], w[1], w[2], w[3]);
    q[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}
// Programmatic dependent launch: let the next kernel in the stream start launching, and
// wait until the previous kernel has completed with its memory visible (a no-op when this
// kernel was launched without the programmatic attribute).
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Block-wide maximum of a non-negative float (blockDim.x a multiple of 32, at most 1024).
__device__ __forceinline__ float block_max(float m, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < static_cast<int>(blockDim.x >> 5) ? s_red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  return m;  // valid in warp 0
}

// One partial max|x| per CTA over rows x cols bf16 (row pitch ldx, cols % 64 == 0), viewed
// as 32-byte chunks: consecutive threads read consecutive chunks, four chunks in flight.
template <bool CONTIG, bool V8>
__global__ void __launch_bounds__(q2cfg::AMAX_THREADS, CONTIG ? 2 : 1) amax_partial_kernel(const uint16_t* __restrict__ x,
                                                                           int64_t rows, int64_t cols, int64_t ldx,
                                                                           float* __restrict__ partial) {
  __shared__ float s_red[32];
  griddep_launch_dependents();  // the quantise kernel waits for this grid's completion anyway
  // normal L2 priority: marking x evict-last was measured 2 us slower on 16384 x 3072 (the
  // quantise kernel, walking the rows backwards, finds what stayed either way)
  const uint64_t keep = l2_policy_evict_normal();
  const int64_t cpr = cols >> 4;  // 32-byte chunks per row
  const int64_t total = rows * cpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  auto addr = [&](int64_t c) -> const uint16_t* {
    if constexpr (CONTIG) {
      return x + c * 16;
    } else {
      const int64_t r = c / cpr;
      return x + r * ldx + (c - r * cpr) * 16;
    }
  };
  uint32_t m = 0u;  // packed |bf16| maxima (max.xorsign.abs leaves a sign that is dropped below)
  int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; c + 3 * stride < total; c += 4 * stride) {
    uint32_t w[4][8];
#pragma unroll
    for (int k = 0; k < 4; ++k) ld_global_32b<V8>(addr(c + k * stride), keep, w[k]);
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int j = 0; j < 8; ++j) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[k][j]));
  }
  for (; c < total; c += stride) {
    uint32_t w[8];
    ld_global_32b<V8>(addr(c), keep, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[j]));
  }
  const float f = fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
  const float b = block_max(f, s_red);
  if (threadIdx.x == 0) partial[blockIdx.x] = b;
}

struct Quant2Args {
  const uint16_t* x;
  int64_t rows, cols, ldx;  // output rows (after the optional interleave) and columns
  int interleave;           // output row 2j <- input row j, 2j+1 <- input row rows/2 + j
  const float* partials;    // amax partials of the first kernel (null: static *gscale)
  int nparts;
  float* gscale;
  uint8_t* codes;           // codes and scales (or null: fake quantisation only)
  uint8_t* sf;
  uint16_t* y;              // quantise-dequantise output in bf16 (or null)
  int64_t ldy;
};

// E2M1 codes of 8 bf16 values (4 packed words) times r: the float32 products are formed two
// at a time (mul.rn.f32x2, each product rounded like a scalar multiply).
__device__ __forceinline__ uint32_t bf16x8_codes(const uint32_t* w, float r) {
  float y[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %4};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(y[2 * j]), "=f"(y[2 * j + 1])
        : "f"(bf16_lo(w[j])), "f"(bf16_hi(w[j])), "f"(r));
  }
  return cvt_e2m1x8(y);
}

// Quantise this lane's 16-value block (8 packed bf16 words): its scale code, 8 bytes of codes
// (0 when the decoded scale is 0), and optionally the dequantised bf16 values.
__device__ __forceinline__ uint32_t quant_lane(const uint32_t (&w)[8], float enc, const float* s_rcp,
                                               uint32_t& lo, uint32_t& hi) {
  const uint32_t s = block_scale_code(bf16x16_amax(w), enc);
  const float r = s_rcp[s];
  lo = bf16x8_codes(w, r);
  hi = bf16x8_codes(w + 4, r);
  if (!(r > 0.0f)) lo = hi = 0u;  // d == 0: every code of the block is 0
  return s;
}

// V8: x (and y) rows start on 32-byte boundaries, so each lane's 16 values move in one
// 256-bit access.
// Task geometry: a warp task is 8 consecutive 64-value groups (512 columns) of one row;
// tpr tasks per row. When tpr <= the number of warps, warp w keeps column chunk w % tpr
// and walks rows w / tpr, + nwarps / tpr, ... (no division in the loop; the few warps past
// (nwarps / tpr) * tpr idle); otherwise every warp walks all rows and column chunks w,
// w + nwarps, ... Rows are walked from the last one up, two per iteration (two loads in
// flight per lane).
// Start of both quantise kernels: wait for the amax partials (or the producer of x), reduce
// them to the tensor's amax and G = amax / (6 * 448) (or read the static G), and fill the
// shared table of the reciprocal of every block scale d = e4m3(s) * G (0 where d is 0; code
// 0x7F is NaN and never produced by the saturating conversion). Returns G.
__device__ __forceinline__ float quant_setup(const Quant2Args& a, float* s_rcp, float* s_red, float* s_G) {
  griddep_wait();  // the amax partials (or the producer of x) are complete and visible
  if (a.partials != nullptr) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < a.nparts; i += blockDim.x) m = fmaxf(m, a.partials[i]);
    m = block_max(m, s_red);
    if (threadIdx.x == 0) {
      const float g = __fdiv_rn(m, kGlobalDiv);
      *s_G = g;
      if (blockIdx.x == 0) *a.gscale = g;
    }
  } else if (threadIdx.x == 0) {
    *s_G = *a.gscale;
  }
  __syncthreads();
  const float G = *s_G;
  if (threadIdx.x < 128) s_rcp[threadIdx.x] = threadIdx.x == 0x7F ? 0.0f : block_inv_scale(threadIdx.x, G);
  __syncthreads();
  return G;
}

template <bool V8>
__global__ void __launch_bounds__(q2cfg::QUANT_THREADS) quantize_rows_kernel(const Quant2Args a) {
  using namespace q2cfg;
  __shared__ float s_rcp[128];
  __shared__ float s_red[32];
  __shared__ float s_G;
  const float G = quant_setup(a, s_rcp, s_red, &s_G);
  const float enc = scale_encode_factor(G);

  const uint64_t stream = l2_policy_evict_first();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane & 3;                        // block of the lane's 64-value group
  const int64_t ng = a.cols >> 6;                  // 64-value groups (scale words) per row
  const int64_t tpr = (ng + 7) >> 3;               // warp tasks per row
  const int64_t rows_pad = (a.rows + 127) & ~int64_t(127);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * QUANT_WARPS;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * QUANT_WARPS + warp;
  int64_t c0, cstep, r0, rstep;
  if (tpr <= nwarps) {
    rstep = nwarps / tpr;
    r0 = w / tpr;
    c0 = w - r0 * tpr;
    cstep = tpr;
    if (r0 >= rstep) return;
  } else {
    c0 = w;
    cstep = nwarps;
    r0 = 0;
    rstep = 1;
  }
  const int64_t half_rows = a.rows >> 1;
  const int64_t code_pitch = a.cols >> 1;
  const int64_t nkb = a.cols >> 4;

  auto src_row = [&](int64_t row) -> int64_t {
    return a.interleave ? ((row & 1) ? half_rows + (row >> 1) : (row >> 1)) : row;
  };
  // scale word of each 64-value group: byte `sub` from lane 4k + sub (0 for padding rows)
  auto store_word = [&](int64_t row, int64_t g, uint32_t s) {
    uint32_t word = s << (8 * sub);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if (a.codes != nullptr && sub == 0 && g < ng) {
      *reinterpret_cast<uint32_t*>(a.sf + sf_word_offset(row, 4 * g, nkb)) = word;
    }
  };
  auto finish = [&](int64_t row, int64_t g, const uint32_t (&wv)[8], bool live) {
    uint32_t s = 0u;
    if (live) {
      uint32_t lo, hi;
      s = quant_lane(wv, enc, s_rcp, lo, hi);
      if (a.codes != nullptr) {
        *reinterpret_cast<uint2*>(a.codes + row * code_pitch + g * 32 + sub * 8) = make_uint2(lo, hi);
      }
      if (a.y != nullptr) {
        uint32_t o[8];
        dequant_block16_bf16(lo, hi, s, G, o);
        st_global_32b<V8>(a.y + row * a.ldy + g * 64 + sub * 16, o);
      }
    }
    store_word(row, g, s);
  };

  for (int64_t gc = c0; gc < tpr; gc += cstep) {
    const int64_t g = gc * 8 + (lane >> 2);
    const bool gl = g < ng;
    int64_t rr = r0;
    for (; rr + rstep < rows_pad; rr += 2 * rstep) {
      const int64_t row0 = rows_pad - 1 - rr, row1 = row0 - rstep;
      const bool l0 = gl && row0 < a.rows, l1 = gl && row1 < a.rows;
      uint32_t w0[8], w1[8];
      if (l0) ld_global_32b<V8>(a.x + src_row(row0) * a.ldx + g * 64 + sub * 16, stream, w0);
      if (l1) ld_global_32b<V8>(a.x + src_row(row1) * a.ldx + g * 64 + sub * 16, stream, w1);
      finish(row0, g, w0, l0);
      finish(row1, g, w1, l1);
    }
    if (rr < rows_pad) {
      const int64_t row0 = rows_pad - 1 - rr;
      const bool l0 = gl && row0 < a.rows;
      uint32_t w0[8];
      if (l0) ld_global_32b<V8>(a.x + src_row(row0) * a.ldx + g * 64 + sub * 16, stream, w0);
      finish(row0, g, w0, l0);
    }
  }
}

// 4 x 4 byte transpose across the 4 lanes of a quad: lane m (m = lane & 3) holds bytes
// M[m][0..3] in `v` and returns M[0..3][m]. Two exchanges: halfwords with lane m ^ 2 (byte
// selectors sel_h: lanes 0-1 keep their low halfword and take the partner's low one, lanes
// 2-3 keep their high halfword and take the partner's high one), then bytes with lane m ^ 1
// (sel_b: even lanes keep bytes 0 and 2, odd lanes bytes 1 and 3).
__device__ __forceinline__ uint32_t quad_transpose_bytes(uint32_t v, uint32_t sel_h, uint32_t sel_b) {
  v = __byte_perm(v, __shfl_xor_sync(0xffffffffu, v, 2), sel_h);
  return __byte_perm(v, __shfl_xor_sync(0xffffffffu, v, 1), sel_b);
}

// Flat form of quantize_rows_kernel, for a contiguous row-major x (ldx == cols) without the
// interleave, x and y (if any, contiguous too) on 32-byte boundaries. x is then one sequence
// of 16-value blocks, and block b's codes sit at byte 8 b of the code array. A warp task is
// 128 consecutive blocks (4 KB of x, 32 scale words): lane i quantises blocks i, 32 + i,
// 64 + i and 96 + i of it (coalesced 256-bit loads), then the lanes of each quad exchange
// their scale bytes so that every lane stores one whole scale word. The row of a lane's
// scale word is tracked incrementally, so the loop has no division. Tasks are walked from
// the end of x, where the amax kernel read last.
// When the amax kernel ran first (a plain launch, so x was complete before either kernel
// started), the first task's loads are issued before the partials are reduced.
// Y: the bf16 quantise-dequantise output y is written too (a.y is not read otherwise).
template <bool Y>
__global__ void __launch_bounds__(q2cfg::QUANT_THREADS, Y ? 3 : 4) quantize_flat_kernel(const Quant2Args a) {
  using namespace q2cfg;
  __shared__ float s_rcp[128];
  __shared__ float s_red[32];
  __shared__ float s_G;
  // x streams past L2 when only codes are written; with the bf16 output y, normal priority
  // was measured faster (16384 x 3072 with amax: 46.8 against 50.3 us)
  const uint64_t stream = Y ? l2_policy_evict_normal() : l2_policy_evict_first();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = a.cols >> 6;        // scale words per row
  const int64_t words = a.rows * ng;     // scale words of the real rows
  const int64_t nblocks = 4 * words;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * QUANT_WARPS;
  int64_t t = ((nblocks + 127) >> 7) - 1 - (static_cast<int64_t>(blockIdx.x) * QUANT_WARPS + warp);
  uint32_t w[4][8];
  auto load_task = [&](int64_t task) {
    const int64_t b0 = 128 * task + lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (b0 + 32 * k < nblocks) ld_global_32b<true>(a.x + (b0 + 32 * k) * 16, stream, w[k]);
    }
  };
  const bool early = a.partials != nullptr;
  if (early && t >= 0) load_task(t);
  const float G = quant_setup(a, s_rcp, s_red, &s_G);
  const float enc = scale_encode_factor(G);

  const int m = lane & 3, q = lane >> 2;
  const int64_t nkb = a.cols >> 4;       // 16-blocks per row
  const int64_t rows_pad = (a.rows + 127) & ~int64_t(127);
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (a.codes != nullptr) {  // the scale words of the padding rows are 0
    for (int64_t pw = words + tid; pw < rows_pad * ng; pw += nthreads) {
      const int64_t row = pw / ng;
      *reinterpret_cast<uint32_t*>(a.sf + sf_word_offset(row, 4 * (pw - row * ng), nkb)) = 0u;
    }
  }
  if (t < 0) return;
  if (!early) load_task(t);
  // this lane's scale word: word 32 t + 8 m + q, i.e. group g of row `row` (g in 32 bits:
  // groups per row are below 2^25); it is a real word while row < rows
  const int64_t wd = 32 * t + 8 * m + q;
  const int ngi = static_cast<int>(ng);
  int64_t row = wd / ng;
  int g = static_cast<int>(wd - row * ng);
  const int64_t wstep = 32 * nwarps;  // scale words per sweep of all warps
  const int64_t drow = wstep / ng;
  const int dg = static_cast<int>(wstep - drow * ng);
  const uint32_t sel_h = m < 2 ? 0x5410u : 0x3276u;
  const uint32_t sel_b = (m & 1) ? 0x3715u : 0x6240u;
  // this lane's first block of task t, and how many blocks from it on are real (only the
  // first task walked, the last of x, can be partial)
  int64_t b0 = 128 * t + lane;
  int64_t rem = nblocks - b0;
  const int64_t bstep = 128 * nwarps;  // blocks per sweep of all warps
  for (bool first = true; t >= 0; t -= nwarps, b0 -= bstep, rem += bstep, first = false) {
    if (!first) load_task(t);
    uint32_t sw = 0u;  // byte k: scale of block b0 + 32 k
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t b = b0 + 32 * k;
      if (32 * k < rem) {
        uint32_t lo, hi;
        const uint32_t s = quant_lane(w[k], enc, s_rcp, lo, hi);
        sw |= s << (8 * k);
        if (a.codes != nullptr) *reinterpret_cast<uint2*>(a.codes + b * 8) = make_uint2(lo, hi);
        if constexpr (Y) {
          uint32_t o[8];
          dequant_block16_bf16(lo, hi, s, G, o);
          st_global_32b<true>(a.y + b * 16, o);
        }
      }
    }
    // lane 4 q + m held byte m of the words of groups 8 k + q; now it holds the word of group
    // 8 m + q (all four of its blocks are real when the word is)
    sw = quad_transpose_bytes(sw, sel_h, sel_b);
    if (a.codes != nullptr && row < a.rows) {
      *reinterpret_cast<uint32_t*>(a.sf + sf_word_offset(row, 4 * g, nkb)) = sw;
    }
    g -= dg;
    row -= drow;
    if (g < 0) {
      g += ngi;
      --row;
    }
  }
}

// (a0, a1) <- (a0 + b0, a1 + b1) and (b0, b1) <- (a0 - b0, a1 - b1): two butterflies with one
// packed add and one packed subtract, each lane rounded like the scalar operation.
__device__ __forceinline__ void butterfly_f32x2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 ra, rb, rs, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 rs, ra, rb;\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rs;\n\t"
      "mov.b64 {%2, %3}, rd;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// =====================================================================================
// MXFP4 (OCP Microscaling: E2M1 elements, one E8M0 scale per 32) with an optional fixed
// block-local transform, the 32-point Walsh-Hadamard matrix H_2 (x) ... (x) H_2 (page
// "KroQuant: efficient post-training quantization for diffusion transformers via
// Kronecker-product structure": an invertible Kronecker-structured transform per block of
// 32 activations; the pages' transforms are learned, this one is fixed). One thread per
// block of 32; lanes 4k..4k+3 hold the 4 blocks of one scale word.
// =====================================================================================
// One block of 32 of row r (block kb) for mx_quantize_kernel: its transform, E8M0 scale and
// codes; the 4 lanes 4k..4k+3 of the calling warp assemble one scale word. Every lane of the
// warp calls it (live = false for lanes past the padded rows).
template <bool V8>
__device__ __forceinline__ void mx_quantize_block(const uint16_t* __restrict__ x, int64_t rows, int64_t ldx,
                                                  int hadamard, int interleave, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, int64_t nb, int64_t r, int64_t kb,
                                                  bool live, int lane, uint64_t stream) {
  const int64_t cols = nb << 5;
  float v[32];
  uint32_t e = 0;
  if (live && r < rows) {
    // with `interleave`, output row 2j reads input row j and 2j+1 reads input row rows/2 + j
    const int64_t src = interleave ? ((r & 1) ? (rows >> 1) + (r >> 1) : (r >> 1)) : r;
    const uint16_t* p = x + src * ldx + kb * 32;
    uint32_t w[16];
    ld_global_32b<V8>(p, stream, *reinterpret_cast<uint32_t(*)[8]>(w));
    ld_global_32b<V8>(p + 16, stream, *reinterpret_cast<uint32_t(*)[8]>(w + 8));
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      v[2 * k] = bf16_lo(w[k]);
      v[2 * k + 1] = bf16_hi(w[k]);
    }
    if (hadamard) {
      // fast Walsh-Hadamard transform, stage h maps (v[j], v[j+h]) to (a + b, a - b), stages
      // h = 1, 2, 4, 8, 16 in that order. In the first four, the butterflies of j and j + 16
      // have the same shape, so one packed add and one packed subtract (two IEEE float32
      // operations each) do both; the last stage pairs j with j + 16 itself.
#pragma unroll
      for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j & h) continue;
          butterfly_f32x2(v[j], v[j + 16], v[j + h], v[j + h + 16]);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float a = v[j], b = v[j + 16];
        v[j] = __fadd_rn(a, b);
        v[j + 16] = __fsub_rn(a, b);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    if (amax > 0.0f) {
      // shared exponent floor(log2(amax)) - 2, clamped to [-127, 127] (a subnormal amax
      // gives -127); scale X = 2^shared, code e = shared + 127
      const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);
      int shared = ex == 0 ? -127 : ex - 127 - 2;
      shared = shared < -127 ? -127 : (shared > 127 ? 127 : shared);
      e = static_cast<uint32_t>(shared + 127);
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - shared) << 23);  // 2^-shared, exact
      float y[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) y[j] = __fmul_rn(v[j], inv);
#pragma unroll
      for (int k = 0; k < 4; ++k) c[k] = cvt_e2m1x8(y + 8 * k);
    }
    *reinterpret_cast<uint4*>(codes + r * (cols >> 1) + kb * 16) = make_uint4(c[0], c[1], c[2], c[3]);
  }
  // the 4 blocks of a scale word sit in lanes 4k..4k+3 (nb % 4 == 0 keeps them in one row)
  uint32_t word = e << (8 * (lane & 3));
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  if (live && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(sf + sf_word_offset(r, kb, nb)) = word;
}

template <bool V8>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ldx, int hadamard, int interleave,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                          float* __restrict__ gscale, float g) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *gscale = g;
  const uint64_t stream = l2_policy_evict_first();
  const int64_t nb = cols >> 5;  // blocks of 32 per row (a multiple of 4)
  const int64_t rows_pad = (rows + 127) & ~int64_t(127);
  const int64_t total = rows_pad * nb;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31;
  // One wave of threads walks the blocks with a stride of the whole grid (a multiple of 32,
  // so the 4 lanes of a scale word stay in one warp); each thread's (row, block) advances
  // by the stride's quotient and remainder, without a division in the loop.
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int64_t r = u0 / nb, kb = u0 - (u0 / nb) * nb;
  const int64_t drow = nthreads / nb, dkb = nthreads - drow * nb;
  for (int64_t base = u0 - lane; base < total; base += nthreads) {
    const bool live = base + lane < total;
    mx_quantize_block<V8>(x, rows, ldx, hadamard, interleave, codes, sf, nb, r, kb, live, lane, stream);
    kb += dkb;
    r += drow;
    if (kb >= nb) {
      kb -= nb;
      ++r;
    }
  }
}

}  // namespace nvfp4
