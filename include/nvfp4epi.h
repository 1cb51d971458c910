/*
 * nvfp4epi — NVFP4 block-scaled GEMM with its follow-on op fused into the epilogue,
 * for NVIDIA B200 (sm_100a). C ABI.
 *
 * What the library computes follows "Serving sub-second Ideogram v4 without quality
 * loss" (fal):
 *   - section "Running the transformer in FP4": FP4 values are E2M1 (1 sign, 2 exponent,
 *     1 mantissa bit) and the matmul runs natively in 4 bits on Blackwell;
 *   - section "Epilogue fusion in brief": the GEMM accumulates a tile on chip, and the
 *     small op that follows (RMSNorm on the attention path, gated SiLU in the FFN) is
 *     applied before the one store of the output, so no second kernel runs;
 *   - sections "Tiles and fragments on Blackwell" / "Why head_dim=256 is hard" /
 *     "Revisit fusion": RMSNorm reduces over a whole head of 128 or 256 columns;
 *   - section "Fusing gated SiLU (SwiGLU)": output = SiLU(C[:, :N/2]) * C[:, N/2:], with
 *     the gate/up weight rows interleaved once at packing time;
 *   - section "Quantization-aware distillation": inference uses static FP4 quantisation,
 *     so the re-quantised output takes a static per-tensor scale.
 * The NVFP4 block format (one unsigned E4M3 scale per 16 elements along K, one FP32
 * scale per tensor) is the format those kernels consume; the page names NVFP4 without
 * spelling out the block size.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller. The library never
 *     allocates device memory.
 *   - Every call is asynchronous on the given stream; nothing synchronises.
 *   - Argument and shape errors return a status synchronously and launch nothing.
 *     CUDA launch errors return NVFP4_ERR_CUDA. There is no exception, no abort and no
 *     device assert. Every wait inside a kernel is bounded in time; a wait that runs
 *     out records NVFP4_ERR_DEVICE_TIMEOUT in a device status word, read with
 *     nvfp4_read_device_status(). The same word holds the one argument error that only
 *     a kernel can see: a misaligned destination in gemm_nvfp4_reduce_rows_f32's device
 *     pointer array (NVFP4_ERR_MISALIGNED).
 *   - Only compute capability 10.0 (B200) is supported (NVFP4_ERR_UNSUPPORTED_DEVICE).
 *   - bf16 tensors are row-major with a leading dimension given in elements.
 */
#ifndef NVFP4EPI_H
#define NVFP4EPI_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, bad flag, inconsistent sizes */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size rule below is not met */
  NVFP4_ERR_MISALIGNED = 3,        /* a pointer or leading dimension is not 16-byte aligned */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 4,
  NVFP4_ERR_CUDA = 5,
  NVFP4_ERR_DEVICE_TIMEOUT = 6
} nvfp4_status;

/*
 * An NVFP4 tensor of rows x cols logical elements, quantised in blocks of 16 adjacent
 * elements along cols (the K axis of a GEMM operand, the N axis of an output).
 *   codes : rows x cols/2 bytes, row-major, row stride cols/2 bytes. Byte j of a row holds
 *           element 2j in bits 0-3 and element 2j+1 in bits 4-7 (E2M1 codes: s e1 e0 m).
 *   sf    : nvfp4_sf_bytes(rows, cols) bytes of unsigned E4M3 block scales in the
 *           tensor-core scale layout: the scales of each 128-row x 4-block tile form one
 *           512-byte unit, units ordered by row tile then by 4-block group, and inside a
 *           unit row r, block c sits at byte (r % 32) * 16 + (r / 32) * 4 + c.
 *   gscale: device pointer to the FP32 per-tensor scale G. Element i of block b decodes
 *           to e2m1(code_i) * e4m3(sf_b) * G.
 */
typedef struct {
  void* codes;
  void* sf;
  float* gscale;
  int64_t rows;
  int64_t cols;
} nvfp4_tensor;

/* Bytes of the block-scale buffer: rows padded to 128, 16-blocks padded to 4. */
int64_t nvfp4_sf_bytes(int64_t rows, int64_t cols);

/* Bytes of device scratch nvfp4_quantize needs when it derives G itself. */
int64_t nvfp4_quantize_workspace_bytes(void);

/* Pack-time row permutation for the SwiGLU weight (section "Fusing gated SiLU"). */
#define NVFP4_SWIGLU_INTERLEAVE 1

/*
 * Activation and weight quantisation ("Serving sub-second Ideogram v4 without quality
 * loss", section "Running the transformer in FP4": E2M1 values; section
 * "Quantization-aware distillation": dynamic or static per-tensor scales).
 * Quantise a bf16 tensor x (rows x cols, leading dimension ldx elements) to NVFP4.
 *   compute_amax = 1: G = amax(|x|) / (6 * 448) is computed on the device and written to
 *                     *out.gscale; `workspace` must hold
 *                     nvfp4_quantize_workspace_bytes() bytes, 4-byte aligned (contents on
 *                     entry ignored: every value the call reads it writes first). It holds
 *                     one partial amax per CTA of the first of two kernels; calls that
 *                     share a workspace must not overlap on the GPU. The first kernel reads
 *                     x once for its amax; the second, launched with programmatic dependent
 *                     launch, reduces the partials and quantises, reading x again from its
 *                     end, where the first kernel read last (that part is likeliest still in
 *                     L2). x rows that start on 32-byte boundaries are read with 256-bit
 *                     accesses.
 *   compute_amax = 0: *out.gscale is used as given (static scale, must be > 0 and finite);
 *                     workspace may be NULL.
 * Per block of 16, in IEEE float32: s = E4M3_rn_satfinite(amax_b * (1 / (6 G))) (s = 0
 * for an all-zero block), d = e4m3(s) * G, q_i = E2M1_rn_satfinite(x_i * (1 / d)) (q = 0
 * when d = 0). These are the decisions of the plain rule (the E4M3 value nearest to
 * amax_b / (6 G), the E2M1 value nearest to x_i / d, ties to even) except where an exact
 * quotient lies within about 2^-21 (relative) of a rounding midpoint: at such a tie the
 * float32 quotient may fall on either side, and either neighbouring code is correct.
 * flags: 0, or NVFP4_SWIGLU_INTERLEAVE: x is a [gate | up] weight of 2*Nh rows and output
 *        row 2j takes input row j, row 2j+1 takes input row Nh + j.
 * Rules: rows >= 1 (even with the interleave flag), cols % 64 == 0, ldx >= cols,
 *        x and ldx*2 bytes 16-byte aligned, out.rows == rows, out.cols == cols,
 *        out.codes 16-byte aligned, out.sf 4-byte aligned. Padding scale bytes are
 *        written as 0.
 */
nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                            int compute_amax, int flags, nvfp4_tensor out,
                            void* workspace, cudaStream_t stream);

/*
 * Fake quantisation (quantise-dequantise) for quantization-aware distillation ("Serving
 * sub-second Ideogram v4 without quality loss", section "Quantization-aware distillation":
 * the forward pass carries the FP4 rounding noise, the backward pass lets the gradient
 * through unchanged, the straight-through estimator, which needs no kernel).
 * y (rows x cols bf16, leading dimension ldy) = bf16(fp32(e2m1(q) * e4m3(s)) * G), where
 * q, s, G are exactly what nvfp4_quantize would produce for x (the level-scale product is
 * exact; the product with G is one fp32 rounding, then round to nearest even bf16).
 *   compute_amax = 1: G = amax(|x|) / (6 * 448) is derived on the device and written to
 *                     *gscale; `workspace` as for nvfp4_quantize.
 *   compute_amax = 0: *gscale is used as given (static scale); workspace may be NULL.
 * Rules: rows >= 1, cols % 64 == 0, ldx >= cols, ldy >= cols, x, y, ldx*2 and ldy*2
 *        bytes 16-byte aligned, gscale 4-byte aligned. y may not overlap x.
 */
nvfp4_status nvfp4_fake_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                 int compute_amax, float* gscale, void* y, int64_t ldy,
                                 void* workspace, cudaStream_t stream);

/*
 * MXFP4 (OCP Microscaling: E2M1 elements, one E8M0 power-of-two scale per 32 values along
 * the columns, no per-tensor scale) with an optional fixed block transform, the 32-point
 * Walsh-Hadamard matrix H32 = H2 (x) H2 (x) H2 (x) H2 (x) H2 ("KroQuant: efficient
 * post-training quantization for diffusion transformers via Kronecker-product structure":
 * an invertible Kronecker-structured transform per block of 32; learned there, fixed here).
 *   flags: MXFP4_HADAMARD32: quantise x H32 (per block of 32, fast Walsh-Hadamard
 *          transform in float32) instead of x. Transform both GEMM operands: (x H)(w H)^T =
 *          32 x w^T, which the per-tensor factor absorbs. NVFP4_SWIGLU_INTERLEAVE: the row
 *          permutation of a [gate | up] weight, as for nvfp4_quantize (rows even).
 *   Per block: shared = clamp(floor(log2(amax)) - 2, -127, 127), scale code e = shared + 127,
 *   q_i = E2M1_rn_satfinite(x_i / 2^shared); an all-zero block has e = 0 and zero codes.
 *   out.codes: rows x cols/2 bytes; out.sf: mxfp4_sf_bytes(rows, cols) bytes in the tensor-
 *   core scale layout counting blocks of 32 (unit = 128 rows x 4 blocks; row r, block c at
 *   (r % 32) * 16 + (r / 32) * 4 + c); *out.gscale is set to the factor a GEMM applies: 1, or
 *   fp32(1/sqrt(32)) with the transform.
 * Rules: cols % 128 == 0, ldx >= cols, x and ldx*2 bytes 16-byte aligned, out.codes 16-byte
 *        and out.sf, out.gscale 4-byte aligned.
 */
#define MXFP4_HADAMARD32 2
int64_t mxfp4_sf_bytes(int64_t rows, int64_t cols);
nvfp4_status mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int flags,
                            nvfp4_tensor out, cudaStream_t stream);

/*
 * GEMM on MXFP4 operands (from mxfp4_quantize; B is N x K): as gemm_nvfp4_pointwise without
 * the NVFP4 output, with the tensor-core MMA kind mxf4nvf4 at block32 (E8M0 scales).
 * alpha = G_A * G_B (1, or 1/32 when both operands carry the transform).
 */
nvfp4_status gemm_mxfp4_pointwise(nvfp4_tensor A, nvfp4_tensor B, const float* bias, int act,
                                  int out_dtype, void* D, int64_t ldd, cudaStream_t stream);
/* D = bf16(G_A G_B acc) on MXFP4 operands. */
nvfp4_status gemm_mxfp4_plain(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                              cudaStream_t stream);
/* gemm_nvfp4_rmsnorm and gemm_nvfp4_swiglu on MXFP4 operands (same arguments and rules; the
 * SwiGLU weight is packed with mxfp4_quantize(..., NVFP4_SWIGLU_INTERLEAVE | ...), and the
 * optional re-quantised output Dq is NVFP4). */
nvfp4_status gemm_mxfp4_rmsnorm(nvfp4_tensor A, nvfp4_tensor B, const float* w, int head_dim,
                                int64_t n_norm_cols, float eps, void* D, int64_t ldd,
                                cudaStream_t stream);
nvfp4_status gemm_mxfp4_swiglu(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                               const nvfp4_tensor* Dq, cudaStream_t stream);

/*
 * Plain epilogue ("Serving sub-second Ideogram v4 without quality loss", section "Epilogue
 * fusion in brief": the accumulator tile is scaled and written once; section "Running the
 * transformer in FP4": the operands stay in 4 bits through the tensor-core MMA).
 * D (M x N bf16, leading dimension ldd) = bf16(G_A * G_B * sum_k A[m,k] * B[n,k]) with
 * A (M x K) and B (N x K) NVFP4, both K-contiguous.
 * Rules: M % 128 == 0, N % 256 == 0, K % 256 == 0, A.cols == B.cols == K,
 *        ldd >= N, ldd % 8 == 0, every pointer 16-byte aligned.
 */
nvfp4_status gemm_nvfp4_plain(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                              cudaStream_t stream);

/*
 * Pointwise epilogue on the plain GEMM ("Serving sub-second Ideogram v4 without quality
 * loss", section "Epilogue fusion in brief": bias, ReLU and cast, each output element on
 * its own):
 *   y[m,n] = act(fma(G_A * G_B, acc[m,n], bias[n]))   (float32; act: none or ReLU)
 *   D = y cast to out_dtype (round to nearest even), and/or
 *   Dq = NVFP4 of bf16(y) with the static scale *Dq->gscale (as nvfp4_quantize with
 *        compute_amax = 0 would give for bf16(y)): the next layer's input.
 *   bias: N float32, 16-byte aligned, or NULL (no bias).
 *   act: NVFP4_ACT_NONE or NVFP4_ACT_RELU.
 *   out_dtype: NVFP4_OUT_BF16, NVFP4_OUT_F16 or NVFP4_OUT_F32; D is M x N of that type with
 *              leading dimension ldd elements (ldd * element size a multiple of 16 bytes),
 *              or NULL.
 *   Dq: M x N NVFP4 (codes 16-byte aligned, scales in the tensor-core layout), or NULL.
 * Shape rules as gemm_nvfp4_plain; D and Dq may not both be NULL.
 */
#define NVFP4_ACT_NONE 0
#define NVFP4_ACT_RELU 1
#define NVFP4_OUT_BF16 0
#define NVFP4_OUT_F16 1
#define NVFP4_OUT_F32 2
nvfp4_status gemm_nvfp4_pointwise(nvfp4_tensor A, nvfp4_tensor B, const float* bias, int act,
                                  int out_dtype, void* D, int64_t ldd, const nvfp4_tensor* Dq,
                                  cudaStream_t stream);

/*
 * Row-parallel GEMM with its reduce-scatter in the epilogue. "Serving sub-second Ideogram v4
 * without quality loss", section "Epilogue fusion in brief", applies the op following a GEMM
 * to the accumulator so that no second pass runs. Here the op is the sum across ranks that
 * follows a GEMM over one rank's slice of K: the down projection of a tensor-parallel FFN
 * block.
 *   C = G_A * G_B * (A B^T)     (float32, M x N, this rank's partial sum)
 *   row m of C is added atomically into  dst[m / rows_per_rank] + (m % rows_per_rank) * ldd,
 *   so destination r receives rows [r * rows_per_rank, (r + 1) * rows_per_rank).
 *   dst: a DEVICE array of `world` float pointers, 8-byte aligned. Each pointer addresses a
 *        rows_per_rank x N float32 block with leading dimension ldd (in floats, a multiple
 *        of 4; pointers 16-byte aligned). A pointer may be another GPU's memory mapped into
 *        this one (peer access); the additions are relaxed atomics at system scope. The host
 *        cannot read the array: a pointer that is not 16-byte aligned is found by the kernel,
 *        which skips that block's rows and records NVFP4_ERR_MISALIGNED for
 *        nvfp4_read_device_status.
 *   The caller zeroes (or seeds) the destinations before the first rank's call, and reads
 *   them only after every rank's call has completed: the call itself synchronises nothing.
 *   Summation order across ranks is unspecified.
 * Rules: the plain rules for A and B; A.rows == world * rows_per_rank, rows_per_rank a
 *        multiple of 128 (UNSUPPORTED_SHAPE otherwise); ldd >= N (INVALID_ARG), ldd % 4 == 0
 *        (MISALIGNED).
 */
nvfp4_status gemm_nvfp4_reduce_rows_f32(nvfp4_tensor A, nvfp4_tensor B, float* const* dst, int world,
                                        int64_t rows_per_rank, int64_t ldd, cudaStream_t stream);

/*
 * Per-head RMSNorm epilogue ("Serving sub-second Ideogram v4 without quality loss",
 * sections "Epilogue fusion in brief" (the formula), "Tiles and fragments on Blackwell" and
 * "Why head_dim=256 is hard" (a head's sum of squares spans more than one thread's
 * fragment), "Revisit fusion").
 * As gemm_nvfp4_plain, then per row and per head of head_dim adjacent columns among the
 * first n_norm_cols: y = x * rsqrt(mean(x^2) + eps) * w[col] (x = G_A G_B acc, float32);
 * columns >= n_norm_cols pass through (the V block of a QKV projection).
 *   w: n_norm_cols float32 weights, one per normalised column (a head_dim-long weight
 *      shared by the heads of a block is expanded by the caller).
 * Rules: the plain rules, head_dim in {128, 256}, n_norm_cols % head_dim == 0,
 *        n_norm_cols <= N, w 16-byte aligned (may be NULL only if n_norm_cols == 0).
 */
nvfp4_status gemm_nvfp4_rmsnorm(nvfp4_tensor A, nvfp4_tensor B, const float* w,
                                int head_dim, int64_t n_norm_cols, float eps,
                                void* D, int64_t ldd, cudaStream_t stream);

/*
 * SwiGLU epilogue ("Serving sub-second Ideogram v4 without quality loss", section "Fusing
 * gated SiLU (SwiGLU)": gate = first half of the weight's rows, gate/up rows interleaved
 * at packing time so each thread holds both; section "Quantization-aware distillation":
 * the optional NVFP4 output uses a static scale). B is the gate|up weight (N = 2*Nh rows)
 * packed with NVFP4_SWIGLU_INTERLEAVE, so accumulator columns come as [g0, u0, g1, u1, ...].
 *   out[m, j] = silu(x_g) * x_u, silu(x) = x / (1 + exp(-x)), x = G_A G_B acc.
 *   D  : M x Nh bf16 output (leading dimension ldd), or NULL.
 *   Dq : M x Nh NVFP4 output quantised from the bf16-rounded values with the static
 *        scale *Dq->gscale (the rule of nvfp4_quantize with compute_amax = 0), or NULL.
 *        Its layout is the A-operand layout of the next GEMM (K = Nh).
 * At least one of D and Dq is given. Rules: the plain rules with Nh = N/2 in place of N
 * for ldd; Dq->rows == M, Dq->cols == Nh.
 */
nvfp4_status gemm_nvfp4_swiglu(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                               const nvfp4_tensor* Dq, cudaStream_t stream);

/*
 * Unfused comparison ops (a GEMM writes its bf16 output; a second kernel applies the op).
 * rmsnorm_heads_bf16: y[:, :n_norm_cols] = per-head RMSNorm of x[:, :n_norm_cols] with
 *   the same formula as gemm_nvfp4_rmsnorm; other columns of y are not touched. y may
 *   equal x (in place). Rules: head_dim in {128, 256}, n_norm_cols % head_dim == 0,
 *   ldx, ldy >= n_norm_cols, 16-byte aligned rows.
 * swiglu_bf16: y (rows x nh) = silu(c[:, :nh]) * c[:, nh:2nh] for c of rows x 2nh
 *   (logical [gate | up] columns). Rules: nh % 8 == 0, ldc >= 2nh, ldy >= nh, 16-byte
 *   aligned rows.
 */
nvfp4_status rmsnorm_heads_bf16(const void* x, int64_t rows, int64_t ldx, const float* w,
                                int head_dim, int64_t n_norm_cols, float eps,
                                void* y, int64_t ldy, cudaStream_t stream);
nvfp4_status swiglu_bf16(const void* c, int64_t rows, int64_t nh, int64_t ldc,
                         void* y, int64_t ldy, cudaStream_t stream);

/*
 * Allocation-free variant of nvfp4_quantize with compute_amax = 1. This entry point has no
 * counterpart on the page; it exists for callers that cannot allocate device memory: code
 * embedded in a host application that owns the whole GPU and hands out only its own
 * buffers (a serving engine that reserves device memory up front), and latency-critical
 * paths where a cudaMalloc, which may synchronise the device, is not acceptable. The caller
 * still provides x and `out`; the scratch the amax reduction needs (one partial maximum per
 * 16384 input values, then the tensor's amax) lives in a 64 KB array of static device
 * memory inside this library, which every GPU that loads the library holds until exit.
 * Results are bit for bit those of nvfp4_quantize(..., compute_amax = 1, ...).
 *   - rows * cols must not exceed NVFP4_NOALLOC_MAX_VALUES, otherwise
 *     NVFP4_ERR_UNSUPPORTED_SHAPE and nothing is launched; the other rules are those of
 *     nvfp4_quantize.
 *   - The first call on a device looks up the array's device address (once per device, with
 *     that device current); make that first call before any stream capture. The address is
 *     kept for the life of the process: do not call this after a cudaDeviceReset of that
 *     device in the same process.
 *   - All calls share the array and leave their values in it. Every value a call reads is
 *     written earlier by the same call, so nothing needs clearing, but calls whose kernels
 *     overlap on the GPU (different streams, or different host threads) race on the array
 *     and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 */
#define NVFP4_NOALLOC_MAX_VALUES 268435456LL /* 16384 partial maxima x 16384 values */
nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                    int flags, nvfp4_tensor out, cudaStream_t stream);

/* Static description of a status code. */
const char* nvfp4_status_string(nvfp4_status status);

/*
 * Synchronise `stream`, return the device status word of the current device (0 or an
 * nvfp4_status recorded by a kernel whose bounded wait ran out) and clear it.
 * Returns -1 if the read itself failed.
 */
int nvfp4_read_device_status(cudaStream_t stream);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a barrier that
 * nothing completes, giving up after limit_ns nanoseconds (1 <= limit_ns <= 1e9).
 * The kernel then records NVFP4_ERR_DEVICE_TIMEOUT in the device status word and
 * returns normally, leaving the context usable.
 */
nvfp4_status nvfp4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream);

/*
 * Barrier of the tensor-parallel FFN-down reduction (the row-parallel GEMM whose epilogue
 * adds its partial rows into the owners' blocks, gemm_nvfp4_reduce_rows_f32; page "Serving
 * sub-second Ideogram v4 without quality loss", section "Epilogue fusion in brief": output
 * tiles are independent, so only this reduction crosses GPUs). One process per GPU; every
 * rank launches it on its stream with the same `epoch`.
 *   signals: device array of `world` pointers; signals[q] is rank q's array of `world`
 *            uint32 words (peer-mapped, e.g. symmetric memory), zeroed once before the
 *            first barrier. signals[rank] is this rank's own array.
 *   epoch:   1, 2, 3, ... one more per barrier (0 is invalid); wraps modulo 2^32.
 * The kernel fences at system scope, writes `epoch` into word [rank] of every rank's
 * array, then waits until every word of its own array has reached `epoch`. A wait longer
 * than limit_ns nanoseconds (1 .. 6e10) gives up: NVFP4_ERR_DEVICE_TIMEOUT is recorded in
 * the device status word (nvfp4_read_device_status) and the kernel returns, leaving the
 * context usable. Argument errors return NVFP4_ERR_INVALID_ARG (or MISALIGNED for an
 * unaligned pointer array) and launch nothing.
 */
nvfp4_status nvfp4_signal_barrier(uint32_t* const* signals, int world, int rank, uint32_t epoch,
                                  int64_t limit_ns, cudaStream_t stream);

/* Number of kernels the library has launched in this process (for launch accounting). */
int64_t nvfp4_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4EPI_H */
