// NVFP4 block-scaled GEMM with a fused epilogue, for sm_100a.
//
// "Serving sub-second Ideogram v4 without quality loss" (fal), section "Epilogue fusion
// in brief": the tensor cores accumulate a tile in TMEM while HBM is not touched for the
// output; the small op is applied to the accumulator and the result is written once.
//
// Two kernels share the epilogue:
//   gemm_nvfp4_pair_kernel  (M > 128) a cluster of 2 CTAs on the two SMs of a TPC runs
//       one 256 x 256 output tile with the pair MMA (tcgen05 cta_group::2): each CTA stages
//       its own 128 rows of A and 128 of the 256 rows of B, so a CTA moves 38 KB per K
//       step of 256 for 128 x 256 x 256 MMA work (5-stage ring). When M % 256 == 128 the
//       last tile's second CTA lies past M: its loads start past the end of A and of its
//       scales and read zeros, its TMA stores are clipped, and its plain stores are skipped.
//   gemm_nvfp4_kernel       (M == 128) one CTA per 128 x 256 tile (3-stage ring).
// Warp roles (512 threads): warps 0-7 epilogue, warp 8 TMA producer, warp 9 TMEM owner
// and MMA issuer, warps 10-13 copy the block scales from shared memory into TMEM
// (tcgen05.cp), warps 14-15 idle. The role warpgroups run on 64 registers a thread and the
// epilogue warpgroups on 184 (setmaxnreg).
// Issue cost sets the main loop's pace. A tcgen05.mma holds up its issuing thread for
// about as long as the tensor pipe takes to run it (M 256 x N 256 x K 64: 128 cycles),
// so the pipe holds about one MMA of backlog at most. Whatever else that thread does
// between two K steps beyond that leaves the pipe idle. So the MMA thread does only this per K step: one wait on the stage's
// barrier, the 4 MMAs and one commit that frees the stage.
// - The scale copies are issued from their own warps, on other SM sub-partitions.
// - The copy warps' commits land on the same stage barrier as the operand bytes, so one
//   wait covers the operand tiles and the scales.
// - A scale slot in TMEM is free again once the stage-empty commit of the step that last
//   used it has arrived.
// - NSLOT (3 or 4) slots let the copies run ahead of the MMAs by NSLOT - 1 steps.
// TMEM holds one 256-column FP32 accumulator at column 0 and the scale slots behind it.
// The MMAs of tile i+1 start once both epilogue warpgroups have moved tile i's
// accumulator into registers.
// Epilogue warp w reads TMEM lanes 32*(w%4).. (its 32 output rows) and columns
// 128*(w/4).. (its half of the 256-column tile); each thread owns one output row.
// Results go through a 128-byte-swizzled staging box and a TMA store.
//
// Epilogues:
//   PLAIN    y = alpha * acc,  alpha = G_A * G_B
//   RMSNORM  per head of 128 or 256 columns (sections "Tiles and fragments on Blackwell",
//            "Why head_dim=256 is hard", "Revisit fusion"): each thread moves its 128
//            accumulator columns into registers and frees the accumulator; a first pass
//            over them sums the squares; a 256-wide head spans the two epilogue
//            warpgroups, which exchange their partial sums through shared memory (an
//            mbarrier, so the wait stays bounded); a second pass over the same registers
//            scales by rstd * w and stores. Columns past n_norm_cols pass through.
//   POINTWISE y = act(alpha * acc + bias[col]) (act: none or ReLU), cast to bf16, f16 or f32
//            (section "Epilogue fusion in brief": bias, ReLU and cast, each element on its
//            own); optional NVFP4 quantisation of bf16(y) with a static scale, the next
//            layer's input.
//   SWIGLU   accumulator columns come interleaved [g0, u0, g1, u1, ...] from the weight
//            packing of section "Fusing gated SiLU (SwiGLU)", so each thread computes
//            silu(g) * u on adjacent columns of its own row; optional NVFP4
//            re-quantisation of the bf16-rounded result with a static scale, one 16-block
//            per 32 accumulator columns.
#pragma once

#include "ptx.cuh"
#include "codec.cuh"
#include "unfused.cuh"

namespace nvfp4 {

enum EpiKind { EPI_PLAIN = 0, EPI_RMSNORM = 1, EPI_SWIGLU = 2, EPI_POINTWISE = 3, EPI_REDUCE = 4 };
enum OutKind { OUT_BF16 = 0, OUT_F16 = 1, OUT_F32 = 2 };

namespace gemm_cfg {
constexpr int BM = 128;                 // output rows per CTA
constexpr int BN = 256;                 // output columns per tile
constexpr int BK = 256;                 // FP4 elements per stage along K
constexpr int BK_BYTES = BK / 2;        // 128: one swizzle row
constexpr int SF_UNIT = 512;            // scales of 128 rows x 64 K
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int COPY_WARPS = 4;
constexpr int ROLE_WARPS = 8;           // two warpgroups: producer, MMA, copy warps, idle
constexpr int NUM_THREADS = EPI_THREADS + 32 * ROLE_WARPS;
constexpr int PRODUCER_WARP = EPI_WARPS;
constexpr int MMA_WARP = EPI_WARPS + 1;
constexpr int COPY_WARP0 = EPI_WARPS + 2;
// Registers per thread after the split: launched with 65536 / 512 = 128 each, the role
// warpgroups drop to ROLE_REGS and the epilogue warpgroups rise to EPI_REGS.
constexpr uint32_t EPI_REGS = 184;
constexpr uint32_t ROLE_REGS = 64;
constexpr uint32_t LAUNCH_REGS = 65536 / NUM_THREADS;
static_assert(2 + COPY_WARPS <= ROLE_WARPS, "warp roles");
static_assert(EPI_THREADS * EPI_REGS + 32 * ROLE_WARPS * ROLE_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr int BOX_BYTES = 32 * 128;     // one staging box: 32 rows x 128 bytes
constexpr int RED_BYTES = 2 * 2 * 128 * 4;
constexpr uint32_t TMEM_COLS = 512;
// The FP32 accumulator takes columns [0, 256); the block scales of one K step take a
// 48-column slot behind it, up to 5 slots (the kernels use 3 or 4).
constexpr uint32_t SF_SLOT0 = 256;
constexpr uint32_t SF_SLOT_COLS = 48;  // per K step: SFA 4 MMAs x 4 columns, then SFB 4 MMAs x 8
constexpr uint32_t SFB_OFF = 16;
constexpr int MAX_SLOTS = 5;
__host__ __device__ constexpr uint32_t sf_slot(uint32_t s) { return SF_SLOT0 + SF_SLOT_COLS * s; }
static_assert(sf_slot(MAX_SLOTS) <= TMEM_COLS, "TMEM plan");
}  // namespace gemm_cfg

// Block-scale format: NVFP4 (E4M3 scale per 16 values) or MXFP4 (E8M0 scale per 32). A
// 512-byte scale unit holds 128 rows x 4 scales, i.e. 64 (NVFP4) or 128 (MXFP4) K values.
template <bool MX>
struct ScaleFmt {
  static constexpr int K_PER_UNIT = MX ? 128 : 64;
  static constexpr int UNITS = gemm_cfg::BK / K_PER_UNIT;  // units per K step per 128 rows: 4 or 2
};

// Shared-memory plan of a kernel with S stages of B_ROWS rows of B per CTA.
template <int S, int B_ROWS, bool MX = false>
struct SmemPlan {
  static constexpr int A_BYTES = gemm_cfg::BM * gemm_cfg::BK_BYTES;                 // 16 KB
  static constexpr int B_BYTES = B_ROWS * gemm_cfg::BK_BYTES;                       // 16 or 32 KB
  static constexpr int SFA_BYTES = ScaleFmt<MX>::UNITS * gemm_cfg::SF_UNIT;         // 2 KB (1 KB MXFP4)
  static constexpr int SFB_BYTES = 2 * ScaleFmt<MX>::UNITS * gemm_cfg::SF_UNIT;     // 4 KB (2 KB MXFP4), 256 rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int OFF_EPI = S * STAGE_BYTES;
  static constexpr int OFF_RED = OFF_EPI + gemm_cfg::EPI_WARPS * gemm_cfg::BOX_BYTES;
  static constexpr int OFF_BAR = OFF_RED + gemm_cfg::RED_BYTES;
  static constexpr int NUM_BARS = 3 * S + 5 + gemm_cfg::COPY_WARPS;  // full, empty, bar_idx, scales loaded
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};
template <bool MX>
using PlanSingleT = SmemPlan<3, 256, MX>;
template <bool MX>
using PlanPairT = SmemPlan<5, 128, MX>;
using PlanSingle = PlanSingleT<false>;
using PlanPair = PlanPairT<false>;

// Barriers past the stage ring (full[S], empty[S]), at empty + S + index.
//   full[s]:  the stage's operand bytes (expect-tx arrival) and one commit per copy warp
//             once the stage's scales are in TMEM
//   empty[s]: one MMA commit when the stage's MMAs are done (frees the stage and the scale
//             slot its step used)
namespace bar_idx {
constexpr int ACC_FULL = 0;   // MMA commit: the tile's accumulator is complete
constexpr int ACC_EMPTY = 1;  // [2] per epilogue warpgroup: accumulator moved to registers
constexpr int RED = 3;
constexpr int DRAIN = 4;      // MMA warp's own drain on give-up
constexpr int CP_DRAIN = 5;   // [COPY_WARPS] copy warps' own drain on give-up
constexpr int SF_LOADED = CP_DRAIN + gemm_cfg::COPY_WARPS;  // [S] a stage's scale units have landed
}  // namespace bar_idx
static_assert(bar_idx::SF_LOADED == 5 + gemm_cfg::COPY_WARPS, "barrier plan");

// Accumulator hand-off between the MMA warp and the epilogue: one "full" barrier (MMA
// commit) and one "empty" barrier per warpgroup (one arrival per warp of that warpgroup,
// in each CTA of the pair).
struct AccBars {
  uint64_t* full;
  uint64_t* empty;  // [2]: empty[wg]
  __device__ __forceinline__ uint64_t* emp(int wg) const { return empty + wg; }
};

// MMA side: tile j may overwrite the accumulator once both warpgroups have read tile j - 1.
__device__ __forceinline__ bool acc_acquire(const AccBars& a, uint32_t j, volatile int* abort_flag,
                                            uint64_t limit, int where) {
  const uint32_t parity = (j & 1u) ^ 1u;
  if (!mbar_wait(a.emp(0), parity, abort_flag, limit, where)) return false;
  if (!mbar_wait(a.emp(1), parity, abort_flag, limit, where)) return false;
  return true;
}

// K steps run by a CTA (or CTA pair) that takes tiles first, first + stride, ...
__device__ __forceinline__ uint32_t ksteps_of(int num_tiles, int K, int first, int stride) {
  const int tiles = first < num_tiles ? (num_tiles - 1 - first) / stride + 1 : 0;
  return static_cast<uint32_t>(tiles) * static_cast<uint32_t>(K / gemm_cfg::BK);
}

// Scale-copy warp `cw` (one elected lane), K step g in ring stage `stage`, scale slot
// g % NSLOT.
// 1. Wait until the stage's scale units have landed. They have their own barrier, so the
//    copies overlap the arrival of the larger code tiles.
// 2. Wait until the slot is free, i.e. the stage-empty commit of step g - NSLOT has
//    arrived. Parity waits on that barrier stay unambiguous while NSLOT <= STAGES: its
//    next completion belongs to step g - NSLOT + STAGES >= g, whose MMAs cannot finish
//    before this step's copies.
// 3. Copy this warp's share of the step's scale units into the slot: 12 units for NVFP4,
//    6 for MXFP4; unit i goes to warp i % COPY_WARPS.
// 4. Commit onto the stage's operand barrier, so that the MMA warp's single wait covers the
//    scales too.
// Slot layout: SFA unit q at columns 4q, SFB rows 0-127 of unit q at 16 + 8q, rows
// 128-255 at 16 + 8q + 4. An NVFP4 unit serves one K = 64 MMA; an MXFP4 unit two (bytes 0-1
// and 2-3 of each word).
// In a CTA pair the leader copies for both CTAs, and the commits go to the leader's
// barriers only. Returns false if a bounded wait gave up, after waiting (bounded) for its
// own copies.
template <bool PAIR, bool MX, int STAGES, int NSLOT, int STAGE_BYTES, int SF_OFF, int SFB_HALF>
__device__ __forceinline__ bool scale_copy_loop(uint8_t* smem, uint64_t* full, uint64_t* bars, uint32_t tmem,
                                                int cw, uint32_t nsteps, volatile int* abort_flag, uint64_t limit,
                                                int where) {
  using namespace gemm_cfg;
  static_assert(NSLOT >= 2 && NSLOT <= STAGES && NSLOT <= MAX_SLOTS, "scale slots");
  uint64_t* empty = full + STAGES;
  uint64_t* sf_loaded = bars + bar_idx::SF_LOADED;
  int stage = 0, slot_i = 0, reuse = 0;  // reuse: stage of step g - NSLOT
  uint32_t phase = 0, reuse_phase = 0;
  bool ok = true;
  for (uint32_t g = 0; g < nsteps; ++g) {
    if (!mbar_wait(&sf_loaded[stage], phase, abort_flag, limit, where) ||
        (g >= static_cast<uint32_t>(NSLOT) && !mbar_wait(&empty[reuse], reuse_phase, abort_flag, limit, where + 1))) {
      ok = false;
      break;
    }
    tc_fence_after();
    constexpr int U = ScaleFmt<MX>::UNITS;
    const uint32_t sfa = smem_u32(smem + stage * STAGE_BYTES) + SF_OFF;
    const uint32_t sfb = sfa + U * SF_UNIT;
    const uint32_t slot = tmem + sf_slot(slot_i);
#pragma unroll
    for (int i = 0; i < 3 * U; ++i) {
      if (i % COPY_WARPS != cw) continue;
      const int q = i / 3, r = i % 3;
      const uint32_t dst = r == 0 ? slot + 4 * q : slot + SFB_OFF + 8 * q + 4 * (r - 1);
      const uint32_t src = r == 0 ? sfa + q * SF_UNIT : sfb + (r - 1) * SFB_HALF + q * SF_UNIT;
      if constexpr (PAIR) {
        tc_copy_scales_pair(dst, smem_desc_scales(src));
      } else {
        tc_copy_scales(dst, smem_desc_scales(src));
      }
    }
    if constexpr (PAIR) {
      tc_commit_pair(&full[stage], 0x1);
    } else {
      tc_commit(&full[stage]);
    }
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1u;
    }
    if (++slot_i == NSLOT) slot_i = 0;
    if (g >= static_cast<uint32_t>(NSLOT)) {  // the next step reuses the slot of step g + 1 - NSLOT
      if (++reuse == STAGES) {
        reuse = 0;
        reuse_phase ^= 1u;
      }
    }
  }
  if (!ok) {
    uint64_t* drain = bars + bar_idx::CP_DRAIN + cw;
    if constexpr (PAIR) {
      tc_commit_pair(drain, 0x1);
    } else {
      tc_commit(drain);
    }
    (void)mbar_wait(drain, 0, nullptr, limit, where + 2);
  }
  return ok;
}

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* ga;
  const float* gb;
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;  // in units of the kernel's tile (128 or 256 rows)
  int n_fastest;                    // tile order: 1 = N index fastest (B stays in L2)
  // RMSNorm
  const float* w;
  int head_dim;
  int n_norm_cols;
  float eps;
  // pointwise
  const float* bias;    // N floats, 16-byte aligned (or null)
  int act;              // 0 none, 1 ReLU
  int out_kind;         // OutKind of D
  // outputs
  int write_d;          // D through tmD (bf16, or out_kind for POINTWISE)
  uint8_t* q_codes;     // NVFP4 quantised output (or null): SwiGLU, POINTWISE
  uint8_t* q_sf;
  const float* q_gscale;
  int q_cols;           // its columns (Nh, or N)
  // row-parallel reduction (EPI_REDUCE): row m of alpha * acc is added into
  // red_dst[m / red_rows] + (m % red_rows) * red_ldd
  float* const* red_dst;
  int64_t red_rows;
  int64_t red_ldd;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void tile_coords(const GemmArgs& a, int t, int& tm, int& tn) {
  if (a.n_fastest) {
    tn = t % a.tiles_n;
    tm = t / a.tiles_n;
  } else {
    tm = t % a.tiles_m;
    tn = t / a.tiles_m;
  }
}

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

// Make the staging box visible to the TMA engine and store it at (x, y). A box whose first
// row is at or past `rows` (the second half of a pair tile that ends past M) is not stored.
__device__ __forceinline__ void flush_box(const CUtensorMap* map, uint8_t* box, int lane, int x, int y,
                                          int rows) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && y < rows) {
    tma_store_2d(map, box, x, y);
    bulk_commit();
  }
}

// Add this warp's staging box (32 rows x 32 floats, 128-byte swizzle) into dst (row pitch ldd
// floats): each instruction adds 4 whole 128-byte rows, 8 lanes per row, 16 bytes a lane.
__device__ __forceinline__ void red_box_f32(const uint8_t* box, int lane, float* dst, int64_t ldd) {
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int idx = it * 32 + lane;
    const int row = idx >> 3, q = idx & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(box + row * 128 + ((q ^ (row & 7)) << 4));
    red_add_v4_f32(dst + static_cast<int64_t>(row) * ldd + 4 * q, v);
  }
  __syncwarp();
}

__device__ __forceinline__ void box_reuse_wait(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

// Per-warp state of the epilogue.
struct EpiCtx {
  const GemmArgs* args;
  const CUtensorMap* tmD;
  uint32_t t_row;     // TMEM address of lane 32*sub, column 0
  int wg, sub, lane;
  uint8_t* box;
  float* red;
  uint64_t* red_bar;
  uint32_t xchg;
  volatile int* abort_flag;
  float alpha, qG, qenc;
};

// Epilogue of one tile: this CTA's 128 rows starting at m0, 256 accumulator columns
// starting at n0. Each thread first moves its 128 accumulator columns from TMEM into
// registers (four 32-column loads, one wait) and calls `release()`, so the MMA warp may
// start the next tile while the op, the rounding and the stores run. Returns false if a
// bounded wait gave up.
template <int EPI, class Release>
__device__ __forceinline__ bool epilogue_tile(EpiCtx& c, int m0, int n0, Release release) {
  using namespace gemm_cfg;
  const GemmArgs& args = *c.args;
  const int lane = c.lane;
  const uint32_t tcol = c.t_row + c.wg * 128;
  const int col0 = n0 + c.wg * 128;
  const int row_in_tile = c.sub * 32 + lane;
  const float alpha = c.alpha;

  uint32_t v[4][32];
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld32(tcol + 32 * q, v[q]);
  tmem_ld_wait();
  release();

  if constexpr (EPI == EPI_SWIGLU) {
    // silu(alpha a) * (alpha b) = (a b) alpha^2 / (1 + 2^(-alpha log2(e) a))
    const float k_exp = -alpha * 1.4426950408889634f;
    const float alpha2 = alpha * alpha;
    uint32_t packed[32];
    uint32_t qc[8];
    uint32_t sfw = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float a = __uint_as_float(v[q][2 * j]);
        const float b = __uint_as_float(v[q][2 * j + 1]);
        o[j] = __fdividef(a * b, 1.0f + ex2_approx(a * k_exp)) * alpha2;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) packed[8 * q + j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
      if (args.q_codes != nullptr) {
        uint32_t lo, hi;
        const uint32_t s = quant_block16_bf16(&packed[8 * q], c.qG, c.qenc, lo, hi);
        qc[2 * q] = lo;
        qc[2 * q + 1] = hi;
        sfw |= s << (8 * q);
      }
    }
    const int oc0 = col0 >> 1;  // first of this thread's 64 output columns
    if (args.write_d) {
      box_reuse_wait(lane);
      stage_row_bf16(c.box, lane, packed);
      flush_box(c.tmD, c.box, lane, oc0, m0 + c.sub * 32, args.M);
    }
    if (args.q_codes != nullptr && m0 < args.M) {
      const int64_t row = m0 + row_in_tile;
      uint4* dst = reinterpret_cast<uint4*>(args.q_codes + row * (args.q_cols >> 1) + (oc0 >> 1));
      dst[0] = make_uint4(qc[0], qc[1], qc[2], qc[3]);
      dst[1] = make_uint4(qc[4], qc[5], qc[6], qc[7]);
      *reinterpret_cast<uint32_t*>(args.q_sf + sf_word_offset(row, oc0 >> 4, args.q_cols >> 4)) = sfw;
    }
    return true;
  } else if constexpr (EPI == EPI_REDUCE) {
    // Row-parallel GEMM with its reduce-scatter fused in: this warp's 32 rows all belong to
    // one destination (red_rows is a multiple of 128), into which alpha * acc is added.
    if (m0 >= args.M) return true;  // the second half of a last pair tile that ends past M
    const int64_t row0 = m0 + c.sub * 32;
    const int64_t owner = row0 / args.red_rows;
    float* const block = args.red_dst[owner];
    // the host cannot see the pointer array: a destination that is not 16-byte aligned is
    // reported in the device status word (NVFP4_ERR_MISALIGNED) and skipped, not dereferenced
    if ((reinterpret_cast<uintptr_t>(block) & 15u) != 0) {
      if (lane == 0) record_status(3, 60);
      return true;
    }
    float* dst = block + (row0 - owner * args.red_rows) * args.red_ldd + col0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[q][j] = __float_as_uint(__fmul_rn(alpha, __uint_as_float(v[q][j])));
      stage_row_bf16(c.box, lane, v[q]);  // 32 words: 32 floats of the row
      red_box_f32(c.box, lane, dst + 32 * q, args.red_ldd);
    }
    return true;
  } else if constexpr (EPI == EPI_POINTWISE) {
    // y = act(alpha * acc + bias[col]) in place of the accumulator bits
    const float4* bp = reinterpret_cast<const float4*>(args.bias + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 b = args.bias != nullptr ? __ldg(bp + 8 * q + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float y = __fmaf_rn(alpha, __uint_as_float(v[q][4 * j4 + e]), bb[e]);
          if (args.act == 1) y = fmaxf(y, 0.0f);
          v[q][4 * j4 + e] = __float_as_uint(y);
        }
      }
    }
    if (args.write_d) {
      if (args.out_kind == OUT_F32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          box_reuse_wait(lane);
          stage_row_bf16(c.box, lane, v[q]);  // 32 words: 32 floats of the row
          flush_box(c.tmD, c.box, lane, col0 + 32 * q, m0 + c.sub * 32, args.M);
        }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t p[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const uint32_t* src = v[2 * h + (j >> 4)];
            const float lo = __uint_as_float(src[2 * (j & 15)]), hi = __uint_as_float(src[2 * (j & 15) + 1]);
            p[j] = args.out_kind == OUT_F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
          }
          box_reuse_wait(lane);
          stage_row_bf16(c.box, lane, p);
          flush_box(c.tmD, c.box, lane, col0 + 64 * h, m0 + c.sub * 32, args.M);
        }
      }
    }
    if (args.q_codes != nullptr && m0 < args.M) {
      const int64_t row = m0 + row_in_tile;
      uint4* dst = reinterpret_cast<uint4*>(args.q_codes + row * (args.q_cols >> 1) + (col0 >> 1));
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        uint32_t sfw = 0u;
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // 32 values: two 16-blocks, 16 bytes of codes
          uint32_t qc[4];
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int blk = 4 * w + 2 * k + hb;
            const uint32_t* src = v[blk >> 1] + 16 * (blk & 1);
            uint32_t p[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              p[j] = pack_bf16x2(__uint_as_float(src[2 * j]), __uint_as_float(src[2 * j + 1]));
            sfw |= quant_block16_bf16(p, c.qG, c.qenc, qc[2 * hb], qc[2 * hb + 1]) << (8 * (2 * k + hb));
          }
          dst[2 * w + k] = make_uint4(qc[0], qc[1], qc[2], qc[3]);
        }
        *reinterpret_cast<uint32_t*>(args.q_sf + sf_word_offset(row, (col0 >> 4) + 4 * w, args.q_cols >> 4)) = sfw;
      }
    }
    return true;
  } else {
    // PLAIN, or RMSNORM (normalised half) / its passthrough half
    bool norm = false;
    float scale = alpha;  // per-row factor applied to acc: alpha, or alpha * rstd
    if constexpr (EPI == EPI_RMSNORM) {
      norm = col0 < args.n_norm_cols;
      if (norm) {
        // sum of squares of the raw accumulator; alpha^2 is applied to the mean
        float ss = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float a = __uint_as_float(v[q][j]);
            ss = fmaf(a, a, ss);
          }
        }
        float mean;
        if (args.head_dim == 256) {
          // the head's other 128 columns sit in the other warpgroup's registers
          float* slot = c.red + (c.xchg & 1u) * 256;
          slot[c.wg * 128 + row_in_tile] = ss;
          mbar_arrive(c.red_bar);
          if (!__all_sync(0xffffffffu, mbar_wait(c.red_bar, c.xchg & 1u, c.abort_flag, args.wait_limit_ns, 5)))
            return false;
          ss = slot[row_in_tile] + slot[128 + row_in_tile];
          ++c.xchg;
          mean = ss * (alpha * alpha * (1.0f / 256.0f));
        } else {
          mean = ss * (alpha * alpha * (1.0f / 128.0f));
        }
        scale = alpha * rsqrtf(mean + args.eps);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t p[32];
      if (EPI == EPI_RMSNORM && norm) {
        const float4* wp = reinterpret_cast<const float4*>(args.w + col0 + 64 * h);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float4 wv = __ldg(wp + j);
          const uint32_t* src = v[2 * h + (j >> 3)];
          const int i = 4 * (j & 7);
          p[2 * j] = pack_bf16x2(__uint_as_float(src[i]) * scale * wv.x, __uint_as_float(src[i + 1]) * scale * wv.y);
          p[2 * j + 1] =
              pack_bf16x2(__uint_as_float(src[i + 2]) * scale * wv.z, __uint_as_float(src[i + 3]) * scale * wv.w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t* src = v[2 * h + (j >> 4)];
          p[j] = pack_bf16x2(alpha * __uint_as_float(src[2 * (j & 15)]), alpha * __uint_as_float(src[2 * (j & 15) + 1]));
        }
      }
      box_reuse_wait(lane);
      stage_row_bf16(c.box, lane, p);
      flush_box(c.tmD, c.box, lane, col0 + 64 * h, m0 + c.sub * 32, args.M);
    }
    return true;
  }
}

__device__ __forceinline__ EpiCtx make_epi_ctx(const GemmArgs& args, const CUtensorMap* tmD, uint32_t tmem,
                                               uint8_t* smem, int off_epi, int off_red, uint64_t* red_bar,
                                               volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5;
  EpiCtx c;
  c.args = &args;
  c.tmD = tmD;
  c.wg = warp >> 2;
  c.sub = warp & 3;
  c.lane = threadIdx.x & 31;
  c.t_row = tmem + (static_cast<uint32_t>(c.sub * 32) << 16);
  c.box = smem + off_epi + warp * gemm_cfg::BOX_BYTES;
  c.red = reinterpret_cast<float*>(smem + off_red);
  c.red_bar = red_bar;
  c.xchg = 0;
  c.abort_flag = abort_flag;
  c.alpha = __fmul_rn(*args.ga, *args.gb);
  c.qG = 0.0f;
  c.qenc = 0.0f;
  if (args.q_codes != nullptr) {
    c.qG = *args.q_gscale;
    c.qenc = scale_encode_factor(c.qG);
  }
  return c;
}

// =====================================================================================
// One CTA per 128 x 256 tile (used when M % 256 == 128)
// =====================================================================================
template <int EPI, bool MX = false>
__global__ void __launch_bounds__(gemm_cfg::NUM_THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmD, const GemmArgs args) {
  using namespace gemm_cfg;
  using P = PlanSingleT<MX>;
  constexpr int U = ScaleFmt<MX>::UNITS;
  constexpr int STAGES = 3;
  constexpr int NSLOT = 3;  // scale slots in TMEM (at most STAGES)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* xbars = empty + STAGES;  // bar_idx layout
  AccBars acc{xbars + bar_idx::ACC_FULL, xbars + bar_idx::ACC_EMPTY};
  uint64_t* red_bar = xbars + bar_idx::RED;
  uint64_t* drain_bar = xbars + bar_idx::DRAIN;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + P::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + COPY_WARPS);  // expect-tx arrival, then one commit per copy warp
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc.full, 1);
    mbar_init(acc.emp(0), EPI_WARPS / 2);
    mbar_init(acc.emp(1), EPI_WARPS / 2);
    mbar_init(red_bar, EPI_THREADS);
    mbar_init(drain_bar, 1);
    for (int w = 0; w < COPY_WARPS; ++w) mbar_init(&xbars[bar_idx::CP_DRAIN + w], 1);
    for (int st = 0; st < STAGES; ++st) mbar_init(&xbars[bar_idx::SF_LOADED + st], 1);
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
  const int64_t kunits = args.K / ScaleFmt<MX>::K_PER_UNIT;  // scale units per 128-row group along K

  if (warp >= EPI_WARPS) {
    regs_release<ROLE_REGS>();
    if (warp == EPI_WARPS) {
      // ------------------------------------------------------------------ producer
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x) {
          int tm, tn;
          tile_coords(args, t, tm, tn);
          for (int kt = 0; kt < ktiles; ++kt) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, limit, 1)) {
              ok = false;
              break;
            }
            uint8_t* sb = smem + stage * P::STAGE_BYTES;
            // scales first, on their own barrier, then the code tiles
            uint64_t* sfl = &xbars[bar_idx::SF_LOADED + stage];
            mbar_arrive_expect_tx(sfl, P::SFA_BYTES + P::SFB_BYTES);
            const int64_t ka = static_cast<int64_t>(kt) * U;
            uint8_t* ssf = sb + P::A_BYTES + P::B_BYTES;
            bulk_load(ssf, args.sfa + (tm * kunits + ka) * SF_UNIT, P::SFA_BYTES, sfl);
            bulk_load(ssf + P::SFA_BYTES, args.sfb + ((2 * tn) * kunits + ka) * SF_UNIT, P::SFB_BYTES / 2, sfl);
            bulk_load(ssf + P::SFA_BYTES + P::SFB_BYTES / 2, args.sfb + ((2 * tn + 1) * kunits + ka) * SF_UNIT,
                      P::SFB_BYTES / 2, sfl);
            mbar_arrive_expect_tx(&full[stage], P::A_BYTES + P::B_BYTES);
            tma_load_2d(sb, &tmA, &full[stage], kt * BK_BYTES, tm * BM);
            tma_load_2d(sb + P::A_BYTES, &tmB, &full[stage], kt * BK_BYTES, tn * BN);
            ++issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) {
          // Tail: wait until the MMAs have released every stage still in use, so that no
          // arrival reaches this CTA's barriers after it exits.
          for (int i = 0; i < STAGES && i < issued; ++i) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, limit, 13)) break;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        } else {
          // Give up: wait (bounded) for the copies this thread started, then leave. The operand
          // barrier also counts the copy warps' commits; a stage whose scale copies were never
          // made keeps it open, and that wait then ends at its limit.
          for (int i = 0; i < STAGES && i < issued; ++i) {
            if (--stage < 0) {
              stage = STAGES - 1;
              phase ^= 1u;
            }
            (void)mbar_wait(&full[stage], phase, nullptr, limit, 11);
            (void)mbar_wait(&xbars[bar_idx::SF_LOADED + stage], phase, nullptr, limit, 11);
          }
        }
      }
    } else if (warp == EPI_WARPS + 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idesc = MX ? idesc_mxfp4(BM, BN, 0) : idesc_nvfp4(BM, BN);
        int stage = 0;
        uint32_t phase = 0, j = 0;
        int sl = 0;  // scale slot of this K step
        bool ok = true;
        // operand descriptors and scale slot advance with the ring instead of being rebuilt
        // from the stage index: fewer instructions in the thread that paces the tensor pipe
        const uint64_t adesc0 = smem_desc_sw128(smem_u32(smem));
        constexpr uint64_t STAGE_DESC = P::STAGE_BYTES >> 4;  // the descriptor's address unit is 16 B
        constexpr uint64_t B_DESC = P::A_BYTES >> 4;
        static_assert((STAGES * P::STAGE_BYTES) >> 4 < (1 << 14), "descriptor address field");
        uint64_t adesc = adesc0;
        uint32_t slot = tmem + sf_slot(0);
        for (int t = blockIdx.x; ok && t < args.num_tiles; t += gridDim.x, ++j) {
          if (!acc_acquire(acc, j, abort_flag, limit, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem;
          for (int kt = 0; kt < ktiles; ++kt) {
            if (!mbar_wait(&full[stage], phase, abort_flag, limit, 3)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t bdesc = adesc + B_DESC;
  #pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              // +32 bytes along K per 64 FP4 values: +2 in the descriptor's address field
              const int u = MX ? kb >> 1 : kb;  // scale unit of this MMA
              const uint32_t id = MX ? (idesc | ((2u * (kb & 1)) << 29) | ((2u * (kb & 1)) << 4)) : idesc;
              tc_mma_nvfp4<MX>(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, id, slot + 4 * u, slot + SFB_OFF + 8 * u,
                               (kt > 0 || kb > 0) ? 1u : 0u);
            }
            tc_commit(&empty[stage]);
            adesc += STAGE_DESC;
            slot += SF_SLOT_COLS;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
              adesc = adesc0;
            }
            if (++sl == NSLOT) {
              sl = 0;
              slot = tmem + sf_slot(0);
            }
          }
          if (!ok) break;
          tc_commit(acc.full);
        }
        if (!ok) {
          tc_commit(drain_bar);
          (void)mbar_wait(drain_bar, 0, nullptr, limit, 12);
        }
      }
    } else if (warp < COPY_WARP0 + COPY_WARPS) {
      // ------------------------------------------------------------------ scale copies
      if (lane == 0) {
        (void)scale_copy_loop<false, MX, STAGES, NSLOT, P::STAGE_BYTES, P::A_BYTES + P::B_BYTES, P::SFB_BYTES / 2>(
            smem, full, xbars, tmem, warp - COPY_WARP0, ksteps_of(args.num_tiles, args.K, blockIdx.x, gridDim.x),
            abort_flag, limit, 14);
      }
    }
  } else {
    regs_acquire<EPI_REGS>();
    // ------------------------------------------------------------------ epilogue
    EpiCtx c = make_epi_ctx(args, &tmD, tmem, smem, P::OFF_EPI, P::OFF_RED, red_bar, abort_flag);
    uint32_t j = 0;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, ++j) {
      int tm, tn;
      tile_coords(args, t, tm, tn);
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc.emp(c.wg));
      };
      // every lane waits; the warp leaves together if any lane gave up
      if (!__all_sync(0xffffffffu, mbar_wait(acc.full, j & 1u, abort_flag, limit, 4))) break;
      tc_fence_after();
      if (!epilogue_tile<EPI>(c, tm * BM, tn * BN, release)) break;
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

// =====================================================================================
// A CTA pair per 256 x 256 tile (used when M % 256 == 0). Cluster of 2 CTAs; CTA rank r
// owns output rows [m0 + 128 r, m0 + 128 r + 128) and stages B rows [n0 + 128 r, +128).
// =====================================================================================
template <int EPI, bool MX = false>
__global__ void __launch_bounds__(gemm_cfg::NUM_THREADS, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                           const __grid_constant__ CUtensorMap tmD, const GemmArgs args) {
  using namespace gemm_cfg;
  using P = PlanPairT<MX>;
  constexpr int U = ScaleFmt<MX>::UNITS;
  constexpr int STAGES = 5;
  constexpr int NSLOT = 4;  // scale slots in TMEM (at most STAGES)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* xbars = empty + STAGES;  // bar_idx layout
  AccBars acc{xbars + bar_idx::ACC_FULL, xbars + bar_idx::ACC_EMPTY};  // leader's empty barriers count both CTAs
  uint64_t* red_bar = xbars + bar_idx::RED;
  uint64_t* drain_bar = xbars + bar_idx::DRAIN;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + P::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = args.wait_limit_ns;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // leader's: one expect-tx arrival for both CTAs' bytes, then one commit per copy warp
      mbar_init(&full[s], 1 + COPY_WARPS);
      mbar_init(&empty[s], 1);  // one multicast commit per use
    }
    mbar_init(acc.full, 1);
    mbar_init(acc.emp(0), EPI_WARPS);  // leader's: one arrival per warp of the warpgroup, per CTA
    mbar_init(acc.emp(1), EPI_WARPS);
    mbar_init(red_bar, EPI_THREADS);
    mbar_init(drain_bar, 1);
    for (int w = 0; w < COPY_WARPS; ++w) mbar_init(&xbars[bar_idx::CP_DRAIN + w], 1);
    for (int st = 0; st < STAGES; ++st) mbar_init(&xbars[bar_idx::SF_LOADED + st], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == EPI_WARPS && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSFA);
    prefetch_tensormap(&tmSFB);
    if (args.write_d) prefetch_tensormap(&tmD);
  }
  // barrier inits visible cluster-wide before any remote arrival or pair allocation
  cluster_sync_all();
  if (warp == EPI_WARPS + 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int ktiles = args.K / BK;
  const int kunits = args.K / ScaleFmt<MX>::K_PER_UNIT;

  if (warp >= EPI_WARPS) {
    regs_release<ROLE_REGS>();
    if (warp == EPI_WARPS) {
      // ------------------------------------------------------------------ producer (both CTAs)
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = cluster_id; ok && t < args.num_tiles; t += num_clusters) {
          int tm, tn;
          tile_coords(args, t, tm, tn);
          const int a_row = tm * 256 + 128 * static_cast<int>(rank);   // this CTA's A rows
          const int b_row = tn * 256 + 128 * static_cast<int>(rank);   // this CTA's half of B
          const int sfa_group = a_row / 128;
          for (int kt = 0; kt < ktiles; ++kt) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, limit, 21)) {
              ok = false;
              break;
            }
            uint8_t* sb = smem + stage * P::STAGE_BYTES;
            // both CTAs' bytes count on the leader's barriers: scales first, on their own
            // barrier, then the code tiles
            uint64_t* sfl = &xbars[bar_idx::SF_LOADED + stage];
            const uint32_t bar_sf = mapa_shared(smem_u32(sfl), 0);
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(sfl, 2 * (P::SFA_BYTES + P::SFB_BYTES));
            // scale units: 512 bytes = 2 rows of the 256-byte-wide scale tensor map
            uint8_t* ssf = sb + P::A_BYTES + P::B_BYTES;
            tma_load_2d_pair(ssf, &tmSFA, bar_sf, 0, 2 * (sfa_group * kunits + U * kt));
            tma_load_2d_pair(ssf + P::SFA_BYTES, &tmSFB, bar_sf, 0, 2 * ((2 * tn) * kunits + U * kt));
            tma_load_2d_pair(ssf + P::SFA_BYTES + P::SFB_BYTES / 2, &tmSFB, bar_sf, 0,
                             2 * ((2 * tn + 1) * kunits + U * kt));
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (P::A_BYTES + P::B_BYTES));
            tma_load_2d_pair(sb, &tmA, bar, kt * BK_BYTES, a_row);
            tma_load_2d_pair(sb + P::A_BYTES, &tmB, bar, kt * BK_BYTES, b_row);
            ++issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) {
          for (int i = 0; i < STAGES && i < issued; ++i) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, limit, 23)) break;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        } else if (leader) {
          // both CTAs' copies complete on the leader's barriers: wait (bounded) for them. The
          // operand barrier also counts the copy warps' commits; a stage whose copies were never
          // made keeps it open, and that wait then ends at its limit.
          for (int i = 0; i < STAGES && i < issued; ++i) {
            if (--stage < 0) {
              stage = STAGES - 1;
              phase ^= 1u;
            }
            (void)mbar_wait(&full[stage], phase, nullptr, limit, 24);
            (void)mbar_wait(&xbars[bar_idx::SF_LOADED + stage], phase, nullptr, limit, 24);
          }
        }
      }
    } else if (warp == EPI_WARPS + 1) {
      // ------------------------------------------------------------------ MMA issuer (leader only)
      if (leader && lane == 0) {
        const uint32_t idesc = MX ? idesc_mxfp4(2 * BM, BN, 0) : idesc_nvfp4(2 * BM, BN);
        int stage = 0;
        uint32_t phase = 0, j = 0;
        int sl = 0;  // scale slot of this K step
        bool ok = true;
        // operand descriptors and scale slot advance with the ring instead of being rebuilt
        // from the stage index: fewer instructions in the thread that paces the tensor pipe
        const uint64_t adesc0 = smem_desc_sw128(smem_u32(smem));
        constexpr uint64_t STAGE_DESC = P::STAGE_BYTES >> 4;  // the descriptor's address unit is 16 B
        constexpr uint64_t B_DESC = P::A_BYTES >> 4;
        static_assert((STAGES * P::STAGE_BYTES) >> 4 < (1 << 14), "descriptor address field");
        uint64_t adesc = adesc0;
        uint32_t slot = tmem + sf_slot(0);
        for (int t = cluster_id; ok && t < args.num_tiles; t += num_clusters, ++j) {
          if (!acc_acquire(acc, j, abort_flag, limit, 22)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem;
          for (int kt = 0; kt < ktiles; ++kt) {
            if (!mbar_wait(&full[stage], phase, abort_flag, limit, 25)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t bdesc = adesc + B_DESC;
  #pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              const int u = MX ? kb >> 1 : kb;  // scale unit of this MMA
              const uint32_t id = MX ? (idesc | ((2u * (kb & 1)) << 29) | ((2u * (kb & 1)) << 4)) : idesc;
              tc_mma_nvfp4_pair<MX>(d_tmem, adesc + 2 * kb, bdesc + 2 * kb, id, slot + 4 * u, slot + SFB_OFF + 8 * u,
                                    (kt > 0 || kb > 0) ? 1u : 0u);
            }
            tc_commit_pair(&empty[stage], 0x3);
            adesc += STAGE_DESC;
            slot += SF_SLOT_COLS;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
              adesc = adesc0;
            }
            if (++sl == NSLOT) {
              sl = 0;
              slot = tmem + sf_slot(0);
            }
          }
          if (!ok) break;
          tc_commit_pair(acc.full, 0x3);
        }
        if (!ok) {
          tc_commit_pair(drain_bar, 0x1);
          (void)mbar_wait(drain_bar, 0, nullptr, limit, 26);
        }
      }
    } else if (warp < COPY_WARP0 + COPY_WARPS) {
      // ------------------------------------------------------------------ scale copies (leader only)
      if (leader && lane == 0) {
        (void)scale_copy_loop<true, MX, STAGES, NSLOT, P::STAGE_BYTES, P::A_BYTES + P::B_BYTES, P::SFB_BYTES / 2>(
            smem, full, xbars, tmem, warp - COPY_WARP0, ksteps_of(args.num_tiles, args.K, cluster_id, num_clusters),
            abort_flag, limit, 31);
      }
    }
  } else {
    regs_acquire<EPI_REGS>();
    // ------------------------------------------------------------------ epilogue (both CTAs)
    EpiCtx c = make_epi_ctx(args, &tmD, tmem, smem, P::OFF_EPI, P::OFF_RED, red_bar, abort_flag);
    uint32_t j = 0;
    for (int t = cluster_id; t < args.num_tiles; t += num_clusters, ++j) {
      int tm, tn;
      tile_coords(args, t, tm, tn);
      const uint32_t leader_empty = mapa_shared(smem_u32(acc.emp(c.wg)), 0);
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_empty);
      };
      if (!__all_sync(0xffffffffu, mbar_wait(acc.full, j & 1u, abort_flag, limit, 27))) break;
      tc_fence_after();
      if (!epilogue_tile<EPI>(c, tm * 256 + 128 * static_cast<int>(rank), tn * BN, release)) break;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  // both CTAs done with each other's barriers and with the pair's TMEM
  cluster_sync_all();
  if (warp == EPI_WARPS + 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace nvfp4
