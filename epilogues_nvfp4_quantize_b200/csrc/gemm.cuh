// NVFP4 block-scaled GEMM with a fused epilogue, for sm_100a.
//
// "Serving sub-second Ideogram v4 without quality loss" (fal), section "Epilogue fusion
// in brief": the tensor cores accumulate a tile in TMEM while HBM is not touched for the
// output; the small op is applied to the accumulator and the result is written once.
//
// Structure (one persistent CTA per SM, 320 threads, warp-specialised):
//   warp 8     TMA producer: A/B code tiles (128-byte swizzle) and their scale units,
//              3-stage shared-memory ring, one mbarrier pair per stage;
//   warp 9     TMEM owner and MMA issuer: copies the stage's E4M3 scales into TMEM
//              (tcgen05.cp) and issues 4 block-scaled MMAs of 128 x 256 x 64 per stage;
//   warps 0-7  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 output rows) and
//              columns 128*(w/4).. (its half of the 256-column tile); each thread owns one
//              output row. Results go through a swizzled staging box and a TMA store.
// Tile = 128 x 256 outputs, K step = 256 (one 128-byte swizzle row of FP4 codes).
//
// Epilogues:
//   PLAIN    y = alpha * acc
//   RMSNORM  per head of 128 or 256 columns (sections "Tiles and fragments on Blackwell",
//            "Why head_dim=256 is hard", "Revisit fusion"): first touch accumulates the
//            sum of squares of the thread's 128 columns; a 256-wide head spans the two
//            epilogue warpgroups, which exchange their partial sums through shared memory
//            (an mbarrier, so the wait stays bounded); second touch re-reads TMEM,
//            scales by rstd * w and stores. Columns past n_norm_cols pass through.
//   SWIGLU   accumulator columns come interleaved [g0, u0, g1, u1, ...] from the weight
//            packing of section "Fusing gated SiLU (SwiGLU)", so each thread computes
//            silu(g) * u on adjacent columns of its own row; optional NVFP4 re-quantisation
//            of the bf16-rounded result with a static scale, 16 outputs per block.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"
#include "unfused.cuh"

namespace nvfp4 {

enum EpiKind { EPI_PLAIN = 0, EPI_RMSNORM = 1, EPI_SWIGLU = 2 };

namespace gemm_cfg {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                 // FP4 elements per stage along K
constexpr int BK_BYTES = BK / 2;        // 128
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK_BYTES;  // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;  // 32 KB
constexpr int SF_UNIT = 512;            // scales of 128 rows x 64 K
constexpr int SFA_BYTES = (BM / 128) * (BK / 64) * SF_UNIT;  // 2 KB
constexpr int SFB_BYTES = (BN / 128) * (BK / 64) * SF_UNIT;  // 4 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int NUM_THREADS = EPI_THREADS + 64;
constexpr int BOX_BYTES = 32 * 128;     // one staging box: 32 rows x 128 bytes
constexpr int OFF_EPI = STAGES * STAGE_BYTES;
constexpr int OFF_RED = OFF_EPI + EPI_WARPS * BOX_BYTES;
constexpr int OFF_BAR = OFF_RED + 2 * 2 * 128 * 4;
constexpr int NUM_BARS = 2 * STAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;    // 256 fp32 columns
constexpr uint32_t SFA_COL = 256;  // 4 MMAs x 4 columns
constexpr uint32_t SFB_COL = 272;  // 4 MMAs x 8 columns
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace gemm_cfg

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* ga;
  const float* gb;
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;
  // RMSNorm
  const float* w;
  int head_dim;
  int n_norm_cols;
  float eps;
  // outputs
  int write_d;          // bf16 output through tmD
  uint8_t* q_codes;     // SwiGLU re-quantised output (or null)
  uint8_t* q_sf;
  const float* q_gscale;
  int q_cols;           // Nh
  uint64_t wait_limit_ns;
};

// Write 64 bf16 values (32 packed words) of this thread's row into the 128-byte-swizzled
// staging box (32 rows x 128 bytes); chunk q of row i goes to chunk q ^ (i % 8).
__device__ __forceinline__ void stage_row_bf16(uint8_t* box, int lane, const uint32_t (&p)[32]) {
  uint8_t* row = box + lane * 128;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 v = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
    *reinterpret_cast<uint4*>(row + ((q ^ (lane & 7)) << 4)) = v;
  }
}

// Make the staging box visible to the TMA engine and store it at (x, y).
__device__ __forceinline__ void flush_box(const CUtensorMap* map, uint8_t* box, int lane, int x, int y) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, box, x, y);
    bulk_commit();
  }
}

__device__ __forceinline__ void box_reuse_wait(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

template <int EPI>
__global__ void __launch_bounds__(gemm_cfg::NUM_THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmD, const GemmArgs args) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* red_bar = acc_full + 2;
  uint64_t* drain_bar = acc_full + 3;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);  // [2 parity][2 wg][128 rows]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, EPI_THREADS);
    mbar_init(red_bar, EPI_THREADS);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == EPI_WARPS && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (args.write_d) prefetch_tensormap(&tmD);
  }
  if (warp == EPI_WARPS + 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int ktiles = args.K / BK;
  const int64_t kunits = args.K / 64;  // scale units per 128-row group along K

  if (warp == EPI_WARPS) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x) {
        const int tm = t % args.tiles_m, tn = t / args.tiles_m;
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, limit, 1)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(sb, &tmA, &full[stage], kt * BK_BYTES, tm * BM);
          tma_load_2d(sb + A_BYTES, &tmB, &full[stage], kt * BK_BYTES, tn * BN);
          const int64_t ka = static_cast<int64_t>(kt) * (BK / 64);
          bulk_load(sb + A_BYTES + B_BYTES, args.sfa + (tm * kunits + ka) * SF_UNIT, SFA_BYTES, &full[stage]);
          bulk_load(sb + A_BYTES + B_BYTES + SFA_BYTES, args.sfb + ((2 * tn) * kunits + ka) * SF_UNIT,
                    SFB_BYTES / 2, &full[stage]);
          bulk_load(sb + A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES / 2,
                    args.sfb + ((2 * tn + 1) * kunits + ka) * SF_UNIT, SFB_BYTES / 2, &full[stage]);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Give up: wait (bounded) for the copies this thread started, then leave.
        for (int i = 0; i < STAGES && i < issued; ++i) {
          if (--stage < 0) {
            stage = STAGES - 1;
            phase ^= 1u;
          }
          (void)mbar_wait(&full[stage], phase, nullptr, limit, 11);
        }
      }
    }
  } else if (warp == EPI_WARPS + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_nvfp4(BM, BN);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag, limit, 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, limit, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          const uint32_t sfa_addr = b_addr + B_BYTES;
          const uint32_t sfb_addr = sfa_addr + SFA_BYTES;
#pragma unroll
          for (int j = 0; j < BK / 64; ++j) {
            tc_copy_scales(tmem + SFA_COL + 4 * j, smem_desc_scales(sfa_addr + j * SF_UNIT));
            tc_copy_scales(tmem + SFB_COL + 8 * j, smem_desc_scales(sfb_addr + j * SF_UNIT));
            tc_copy_scales(tmem + SFB_COL + 8 * j + 4, smem_desc_scales(sfb_addr + SFB_BYTES / 2 + j * SF_UNIT));
          }
          const uint64_t adesc = smem_desc_sw128(a_addr);
          const uint64_t bdesc = smem_desc_sw128(b_addr);
#pragma unroll
          for (int kb = 0; kb < BK / 64; ++kb) {
            // +32 bytes along K per 64 FP4 values: +2 in the descriptor's address field
            tc_mma_nvfp4(tmem + ACC_COL, adesc + 2 * kb, bdesc + 2 * kb, idesc, tmem + SFA_COL + 4 * kb,
                         tmem + SFB_COL + 8 * kb, (kt > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      if (!ok) {
        tc_commit(drain_bar);
        (void)mbar_wait(drain_bar, 0, nullptr, limit, 12);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int wg = warp >> 2;          // column half of the tile
    const int sub = warp & 3;          // TMEM lane quadrant = output row group
    const int row_in_tile = sub * 32 + lane;
    uint8_t* box = smem + OFF_EPI + warp * BOX_BYTES;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const float alpha = __fmul_rn(*args.ga, *args.gb);
    float qG = 0.0f, qenc = 0.0f;
    if (EPI == EPI_SWIGLU && args.q_codes != nullptr) {
      qG = *args.q_gscale;
      qenc = scale_encode_factor(qG);
    }
    uint32_t acc_phase = 0, xchg = 0;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
      const int tm = t % args.tiles_m, tn = t / args.tiles_m;
      const int m0 = tm * BM, n0 = tn * BN;
      // every lane waits; the warp leaves together if any lane gave up
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, acc_phase, abort_flag, limit, 4))) break;
      tc_fence_after();
      const uint32_t tcol = t_row + ACC_COL + wg * 128;
      const int col0 = n0 + wg * 128;

      if constexpr (EPI == EPI_SWIGLU) {
        uint32_t packed[32];
        uint32_t qc[8];
        uint32_t sfw = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v[32];
          tmem_ld32(tcol + 32 * q, v);
          tmem_ld_wait();
          if (q == 3) {
            tc_fence_before();
            mbar_arrive(acc_empty);
          }
          float o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float g = alpha * __uint_as_float(v[2 * j]);
            const float u = alpha * __uint_as_float(v[2 * j + 1]);
            o[j] = silu_f32(g) * u;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) packed[8 * q + j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
          if (args.q_codes != nullptr) {
            float ob[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              ob[2 * j] = bf16_lo(packed[8 * q + j]);
              ob[2 * j + 1] = bf16_hi(packed[8 * q + j]);
            }
            uint32_t lo, hi;
            const uint32_t s = quant_block16(ob, qG, qenc, lo, hi);
            qc[2 * q] = lo;
            qc[2 * q + 1] = hi;
            sfw |= s << (8 * q);
          }
        }
        const int oc0 = col0 >> 1;  // first of this thread's 64 output columns
        if (args.write_d) {
          box_reuse_wait(lane);
          stage_row_bf16(box, lane, packed);
          flush_box(&tmD, box, lane, oc0, m0 + sub * 32);
        }
        if (args.q_codes != nullptr) {
          const int64_t row = m0 + row_in_tile;
          uint4* dst = reinterpret_cast<uint4*>(args.q_codes + row * (args.q_cols >> 1) + (oc0 >> 1));
          dst[0] = make_uint4(qc[0], qc[1], qc[2], qc[3]);
          dst[1] = make_uint4(qc[4], qc[5], qc[6], qc[7]);
          *reinterpret_cast<uint32_t*>(args.q_sf + sf_word_offset(row, oc0 >> 4, args.q_cols >> 4)) = sfw;
        }
      } else {
        // PLAIN, or RMSNORM (normalised half) / its passthrough half
        bool norm = false;
        float rstd = 1.0f;
        if constexpr (EPI == EPI_RMSNORM) {
          norm = col0 < args.n_norm_cols;
          if (norm) {
            float ss = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
              uint32_t v0[32], v1[32];
              tmem_ld32(tcol + 32 * q, v0);
              tmem_ld32(tcol + 32 * q + 32, v1);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float a = alpha * __uint_as_float(v0[j]);
                const float b = alpha * __uint_as_float(v1[j]);
                ss = fmaf(a, a, ss);
                ss = fmaf(b, b, ss);
              }
            }
            float mean;
            if (args.head_dim == 256) {
              float* slot = red + (xchg & 1u) * 256;
              slot[wg * 128 + row_in_tile] = ss;
              mbar_arrive(red_bar);
              if (!__all_sync(0xffffffffu, mbar_wait(red_bar, xchg & 1u, abort_flag, limit, 5))) break;
              ss = slot[row_in_tile] + slot[128 + row_in_tile];
              ++xchg;
              mean = ss * (1.0f / 256.0f);
            } else {
              mean = ss * (1.0f / 128.0f);
            }
            rstd = rsqrtf(mean + args.eps);
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v0[32], v1[32];
          tmem_ld32(tcol + 64 * h, v0);
          tmem_ld32(tcol + 64 * h + 32, v1);
          tmem_ld_wait();
          if (h == 1) {
            tc_fence_before();
            mbar_arrive(acc_empty);
          }
          uint32_t p[32];
          if (EPI == EPI_RMSNORM && norm) {
            const float* wp = args.w + col0 + 64 * h;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float2 wa = __ldg(reinterpret_cast<const float2*>(wp + 2 * j));
              const float2 wb = __ldg(reinterpret_cast<const float2*>(wp + 32 + 2 * j));
              p[j] = pack_bf16x2(alpha * __uint_as_float(v0[2 * j]) * rstd * wa.x,
                                 alpha * __uint_as_float(v0[2 * j + 1]) * rstd * wa.y);
              p[16 + j] = pack_bf16x2(alpha * __uint_as_float(v1[2 * j]) * rstd * wb.x,
                                      alpha * __uint_as_float(v1[2 * j + 1]) * rstd * wb.y);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              p[j] = pack_bf16x2(alpha * __uint_as_float(v0[2 * j]), alpha * __uint_as_float(v0[2 * j + 1]));
              p[16 + j] = pack_bf16x2(alpha * __uint_as_float(v1[2 * j]), alpha * __uint_as_float(v1[2 * j + 1]));
            }
          }
          box_reuse_wait(lane);
          stage_row_bf16(box, lane, p);
          flush_box(&tmD, box, lane, col0 + 64 * h, m0 + sub * 32);
        }
      }
      acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == EPI_WARPS + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace nvfp4
