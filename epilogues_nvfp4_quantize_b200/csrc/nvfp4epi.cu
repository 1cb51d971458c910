// C-ABI entry points of libnvfp4epi: argument validation, tensor-map encoding and
// kernel launches. All device code is in the included headers, built as one
// translation unit for sm_100a.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "nvfp4epi.h"
#include "ptx.cuh"
#include "codec.cuh"
#include "quantize.cuh"
#include "unfused.cuh"
#include "gemm.cuh"

#define NVFP4_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxDevices = 64;

std::atomic<int64_t> g_launches{0};
constexpr int kEpiKinds = nvfp4::EPI_REDUCE + 1;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  // per kernel instance: index epilogue kind + kEpiKinds * (MXFP4 scales)
  bool gemm_attr_set[2 * kEpiKinds] = {};
  bool pair_attr_set[2 * kEpiKinds] = {};
  int pair_clusters[2 * kEpiKinds] = {};
  // resident CTAs of quantize_rows_kernel<V8 = false>, <V8 = true>, quantize_flat_kernel<Y =
  // false>, <Y = true>
  int quant_ctas_per_sm[4] = {0, 0, 0, 0};
  int mx_ctas_per_sm[2] = {0, 0};  // resident CTAs of mx_quantize_kernel<V8 = false, true>
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

nvfp4_status current_device(int* dev_out, DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
    d.probed = true;
  }
  if (!d.supported) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  *dev_out = dev;
  *info = &d;
  return NVFP4_OK;
}

nvfp4_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The GEMM kernels split their registers between warpgroups at run time (setmaxnreg): the
// epilogue warpgroups can only grow if the block was launched with enough registers for
// the whole split, otherwise they would wait forever. Checked once per kernel, before its
// first launch.
template <class Kernel>
bool register_split_fits(Kernel kern) {
  using namespace nvfp4::gemm_cfg;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
  const long long launched = static_cast<long long>(fa.numRegs) * NUM_THREADS;
  const long long needed = static_cast<long long>(EPI_THREADS) * EPI_REGS + 32ll * ROLE_WARPS * ROLE_REGS;
  return launched >= needed;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

nvfp4_status check_operand(const nvfp4_tensor& t) {
  if (t.codes == nullptr || t.sf == nullptr || t.gscale == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (t.rows <= 0 || t.cols <= 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(t.codes) || !aligned16(t.sf)) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

// Common checks and launch of the GEMM kernels: the CTA-pair kernel from M = 256 on (for
// M % 256 == 128 its last tile's second CTA computes rows past M, which are zeros and are
// not stored), the single-CTA kernel for M = 128.
template <int EPI, bool MX = false>
nvfp4_status run_gemm(const nvfp4_tensor& A, const nvfp4_tensor& B, void* D, int64_t ldd, int64_t n_out,
                      nvfp4::GemmArgs args, cudaStream_t stream) {
  using namespace nvfp4::gemm_cfg;
  nvfp4_status st;
  if ((st = check_operand(A)) != NVFP4_OK) return st;
  if ((st = check_operand(B)) != NVFP4_OK) return st;
  const int64_t M = A.rows, K = A.cols, N = B.rows;
  if (B.cols != K) return NVFP4_ERR_INVALID_ARG;
  if (M % BM || N % BN || K % BK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const int out_kind = EPI == nvfp4::EPI_POINTWISE ? args.out_kind : nvfp4::OUT_BF16;
  const int esize = out_kind == nvfp4::OUT_F32 ? 4 : 2;
  if (D != nullptr) {
    if (ldd < n_out) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(D) || (ldd * esize) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  }
  int dev;
  DeviceInfo* info;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;

  const bool pair = M > BM;
  CUtensorMap tmA, tmB, tmD, tmSFA, tmSFB;
  std::memset(&tmD, 0, sizeof(tmD));
  if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A.codes, K / 2, M, K / 2, BK_BYTES, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B.codes, K / 2, N, K / 2, BK_BYTES, pair ? 128 : BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ERR_CUDA;
  if (pair) {
    // the block scales seen as rows of 256 bytes; one 128-row x 256-K group = 8 rows
    // (NVFP4, a scale per 16 values) or 4 rows (MXFP4, a scale per 32)
    const int64_t per_scale = MX ? 32 : 16;
    const uint32_t box_rows = MX ? 4 : 8;
    if (!make_map_2d(&tmSFA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A.sf, 256, M * (K / per_scale) / 256, 256, 256, box_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&tmSFB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B.sf, 256, N * (K / per_scale) / 256, 256, 256, box_rows,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return NVFP4_ERR_CUDA;
  }
  // D staged by 32 rows x 128 bytes and stored by TMA: 64 columns of bf16/f16 or 32 of f32
  const CUtensorMapDataType d_type = out_kind == nvfp4::OUT_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                     : out_kind == nvfp4::OUT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (D != nullptr && !make_map_2d(&tmD, d_type, D, n_out, M, ldd * esize, 128 / esize, 32,
                                   CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ERR_CUDA;

  args.sfa = static_cast<const uint8_t*>(A.sf);
  args.sfb = static_cast<const uint8_t*>(B.sf);
  args.ga = A.gscale;
  args.gb = B.gscale;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.tiles_m = static_cast<int>(pair ? (M + 255) / 256 : M / BM);
  args.tiles_n = static_cast<int>(N / BN);
  args.num_tiles = args.tiles_m * args.tiles_n;
  // keep the smaller operand resident in L2 while the larger one streams through once
  args.n_fastest = N <= M ? 1 : 0;
  args.write_d = D != nullptr;
  args.wait_limit_ns = kWaitLimitNs;

  if (!pair) {
    using P = nvfp4::PlanSingleT<MX>;
    auto kern = nvfp4::gemm_nvfp4_kernel<EPI, MX>;
    {
      std::lock_guard<std::mutex> lock(g_mutex);
      if (!info->gemm_attr_set[EPI + kEpiKinds * MX]) {
        if (!register_split_fits(kern)) return NVFP4_ERR_CUDA;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM_BYTES) != cudaSuccess)
          return NVFP4_ERR_CUDA;
        info->gemm_attr_set[EPI + kEpiKinds * MX] = true;
      }
    }
    const int grid = args.num_tiles < info->sm_count ? args.num_tiles : info->sm_count;
    kern<<<grid, NUM_THREADS, P::SMEM_BYTES, stream>>>(tmA, tmB, tmD, args);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return launch_status();
  }

  using P = nvfp4::PlanPairT<MX>;
  auto kern = nvfp4::gemm_nvfp4_pair_kernel<EPI, MX>;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = P::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!info->pair_attr_set[EPI + kEpiKinds * MX]) {
      if (!register_split_fits(kern)) return NVFP4_ERR_CUDA;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM_BYTES) != cudaSuccess)
        return NVFP4_ERR_CUDA;
      cfg.gridDim = dim3(2 * (info->sm_count / 2), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return NVFP4_ERR_CUDA;
      info->pair_clusters[EPI + kEpiKinds * MX] = n;
      info->pair_attr_set[EPI + kEpiKinds * MX] = true;
    }
    max_clusters = info->pair_clusters[EPI + kEpiKinds * MX];
  }
  const int clusters = args.num_tiles < max_clusters ? args.num_tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmSFA, tmSFB, tmD, args) != cudaSuccess) return NVFP4_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

}  // namespace

// Launch of the two-kernel quantiser (quantize.cuh) for nvfp4_quantize and
// nvfp4_fake_quantize: with compute_amax, the amax partials kernel then the quantise kernel
// (programmatic dependent launch); with a static scale, the quantise kernel alone.
static nvfp4_status launch_quantize2(DeviceInfo* info, const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                     int compute_amax, bool inter, float* gscale, uint8_t* codes, uint8_t* sf,
                                     uint16_t* y, int64_t ldy, void* workspace, cudaStream_t stream) {
  using namespace nvfp4::q2cfg;
  const uint16_t* xp = static_cast<const uint16_t*>(x);
  // 256-bit accesses need every row of x (and of y) to start on a 32-byte boundary
  const bool x_v8 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  const bool y_v8 = y == nullptr || ((reinterpret_cast<uintptr_t>(y) & 31u) == 0 && (ldy % 16) == 0);
  nvfp4::Quant2Args qa{};
  qa.x = xp;
  qa.rows = rows;
  qa.cols = cols;
  qa.ldx = ldx;
  qa.interleave = inter ? 1 : 0;
  qa.gscale = gscale;
  qa.codes = codes;
  qa.sf = sf;
  qa.y = y;
  qa.ldy = ldy;
  if (compute_amax) {
    const int64_t chunks = rows * (cols / 16);
    int64_t parts = (chunks + 4 * AMAX_THREADS - 1) / (4 * AMAX_THREADS);
    const int64_t cap = 2ll * info->sm_count < MAX_PARTIALS ? 2ll * info->sm_count : MAX_PARTIALS;
    if (parts > cap) parts = cap;
    if (parts < 1) parts = 1;
    float* partials = static_cast<float*>(workspace);
    const dim3 grid(static_cast<unsigned>(parts));
    if (ldx == cols && x_v8) {
      nvfp4::amax_partial_kernel<true, true><<<grid, AMAX_THREADS, 0, stream>>>(xp, rows, cols, ldx, partials);
    } else if (ldx == cols) {
      nvfp4::amax_partial_kernel<true, false><<<grid, AMAX_THREADS, 0, stream>>>(xp, rows, cols, ldx, partials);
    } else if (x_v8) {
      nvfp4::amax_partial_kernel<false, true><<<grid, AMAX_THREADS, 0, stream>>>(xp, rows, cols, ldx, partials);
    } else {
      nvfp4::amax_partial_kernel<false, false><<<grid, AMAX_THREADS, 0, stream>>>(xp, rows, cols, ldx, partials);
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    nvfp4_status st;
    if ((st = launch_status()) != NVFP4_OK) return st;
    qa.partials = partials;
    qa.nparts = static_cast<int>(parts);
  }
  const bool v8 = x_v8 && y_v8;
  // the flat kernel: x (and y) contiguous and 32-byte aligned, no interleave
  const bool flat = v8 && !inter && ldx == cols && (y == nullptr || ldy == cols);
  const int kind = flat ? (y != nullptr ? 3 : 2) : (v8 ? 1 : 0);
  {
    // CTAs that fit on an SM at once: the kernel's warps stride over the whole tensor, so a
    // grid larger than one wave would only queue CTAs behind it
    std::lock_guard<std::mutex> lock(g_mutex);
    int& per_sm = info->quant_ctas_per_sm[kind];
    if (per_sm == 0) {
      int n = 0;
      const cudaError_t e =
          kind == 3   ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quantize_flat_kernel<true>,
                                                                      QUANT_THREADS, 0)
          : kind == 2 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quantize_flat_kernel<false>,
                                                                      QUANT_THREADS, 0)
          : kind == 1
              ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quantize_rows_kernel<true>, QUANT_THREADS, 0)
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quantize_rows_kernel<false>, QUANT_THREADS, 0);
      if (e != cudaSuccess || n < 1) return NVFP4_ERR_CUDA;
      per_sm = n;
    }
  }
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  // warp tasks: 128 blocks of 16 (flat), or 512 columns of one row (row kernel)
  const int64_t tasks = flat ? (rows * (cols / 16) + 127) / 128 : rows_pad * ((cols / 64 + 7) / 8);
  int64_t grid = (tasks + QUANT_WARPS - 1) / QUANT_WARPS;
  const int64_t full = static_cast<int64_t>(info->quant_ctas_per_sm[kind]) * info->sm_count;
  if (grid > full) grid = full;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(QUANT_THREADS, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = kind == 3   ? cudaLaunchKernelEx(&cfg, nvfp4::quantize_flat_kernel<true>, qa)
                        : kind == 2 ? cudaLaunchKernelEx(&cfg, nvfp4::quantize_flat_kernel<false>, qa)
                        : kind == 1 ? cudaLaunchKernelEx(&cfg, nvfp4::quantize_rows_kernel<true>, qa)
                                    : cudaLaunchKernelEx(&cfg, nvfp4::quantize_rows_kernel<false>, qa);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

NVFP4_API int64_t nvfp4_sf_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return -1;
  return ((rows + 127) / 128) * 128 * ((cols / 16 + 3) / 4) * 4;
}

NVFP4_API int64_t nvfp4_quantize_workspace_bytes(void) {
  return nvfp4::q2cfg::MAX_PARTIALS * static_cast<int64_t>(sizeof(float));
}

NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int compute_amax,
                                      int flags, nvfp4_tensor out, void* workspace, cudaStream_t stream) {
  if (x == nullptr || out.codes == nullptr || out.sf == nullptr || out.gscale == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (compute_amax != 0 && compute_amax != 1) return NVFP4_ERR_INVALID_ARG;
  if (compute_amax && workspace == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (flags & ~NVFP4_SWIGLU_INTERLEAVE) return NVFP4_ERR_INVALID_ARG;
  if (out.rows != rows || out.cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || cols % 64 != 0 || ldx < cols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((flags & NVFP4_SWIGLU_INTERLEAVE) && (rows % 2) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > (1ll << 31) || cols > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx % 8) != 0 || !aligned16(out.codes) ||
      (reinterpret_cast<uintptr_t>(out.sf) & 3u) != 0 ||
      (compute_amax && (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;

  return launch_quantize2(info, x, rows, cols, ldx, compute_amax, (flags & NVFP4_SWIGLU_INTERLEAVE) != 0,
                          out.gscale, static_cast<uint8_t*>(out.codes), static_cast<uint8_t*>(out.sf), nullptr, 0,
                          workspace, stream);
}

NVFP4_API nvfp4_status nvfp4_fake_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int compute_amax,
                                           float* gscale, void* y, int64_t ldy, void* workspace,
                                           cudaStream_t stream) {
  if (x == nullptr || y == nullptr || gscale == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (compute_amax != 0 && compute_amax != 1) return NVFP4_ERR_INVALID_ARG;
  if (compute_amax && workspace == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || cols % 64 != 0 || ldx < cols || ldy < cols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > (1ll << 31) || cols > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx % 8) != 0 || !aligned16(y) || (ldy % 8) != 0 ||
      (reinterpret_cast<uintptr_t>(gscale) & 3u) != 0 ||
      (compute_amax && (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0))
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  return launch_quantize2(info, x, rows, cols, ldx, compute_amax, false, gscale, nullptr, nullptr,
                          static_cast<uint16_t*>(y), ldy, workspace, stream);
}

NVFP4_API nvfp4_status gemm_nvfp4_plain(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                                        cudaStream_t stream) {
  if (D == nullptr) return NVFP4_ERR_INVALID_ARG;
  nvfp4::GemmArgs args{};
  return run_gemm<nvfp4::EPI_PLAIN>(A, B, D, ldd, B.rows, args, stream);
}

NVFP4_API nvfp4_status gemm_nvfp4_pointwise(nvfp4_tensor A, nvfp4_tensor B, const float* bias, int act,
                                            int out_dtype, void* D, int64_t ldd, const nvfp4_tensor* Dq,
                                            cudaStream_t stream) {
  if (D == nullptr && Dq == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_RELU) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
    return NVFP4_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return NVFP4_ERR_MISALIGNED;
  nvfp4::GemmArgs args{};
  args.bias = bias;
  args.act = act;
  args.out_kind = out_dtype;
  if (Dq != nullptr) {
    if (Dq->codes == nullptr || Dq->sf == nullptr || Dq->gscale == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (Dq->rows != A.rows || Dq->cols != B.rows) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(Dq->codes) || !aligned16(Dq->sf)) return NVFP4_ERR_MISALIGNED;
    args.q_codes = static_cast<uint8_t*>(Dq->codes);
    args.q_sf = static_cast<uint8_t*>(Dq->sf);
    args.q_gscale = Dq->gscale;
    args.q_cols = static_cast<int>(B.rows);
  }
  return run_gemm<nvfp4::EPI_POINTWISE>(A, B, D, ldd, B.rows, args, stream);
}

NVFP4_API nvfp4_status gemm_nvfp4_reduce_rows_f32(nvfp4_tensor A, nvfp4_tensor B, float* const* dst, int world,
                                                  int64_t rows_per_rank, int64_t ldd, cudaStream_t stream) {
  if (dst == nullptr || (reinterpret_cast<uintptr_t>(dst) & 7u) != 0) return NVFP4_ERR_INVALID_ARG;
  if (world < 1 || rows_per_rank <= 0) return NVFP4_ERR_INVALID_ARG;
  if (rows_per_rank % 128 != 0 || A.rows != static_cast<int64_t>(world) * rows_per_rank)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ldd < B.rows) return NVFP4_ERR_INVALID_ARG;
  if (ldd % 4 != 0) return NVFP4_ERR_MISALIGNED;
  nvfp4::GemmArgs args{};
  args.red_dst = dst;
  args.red_rows = rows_per_rank;
  args.red_ldd = ldd;
  return run_gemm<nvfp4::EPI_REDUCE>(A, B, nullptr, 0, B.rows, args, stream);
}

NVFP4_API int64_t mxfp4_sf_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return -1;
  return ((rows + 127) / 128) * 128 * ((cols / 32 + 3) / 4) * 4;
}

NVFP4_API nvfp4_status mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ldx, int flags,
                                      nvfp4_tensor out, cudaStream_t stream) {
  if (x == nullptr || out.codes == nullptr || out.sf == nullptr || out.gscale == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (flags & ~(MXFP4_HADAMARD32 | NVFP4_SWIGLU_INTERLEAVE)) return NVFP4_ERR_INVALID_ARG;
  if ((flags & NVFP4_SWIGLU_INTERLEAVE) && (rows % 2) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (out.rows != rows || out.cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || cols % 128 != 0 || ldx < cols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > (1ll << 31) || cols > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx % 8) != 0 || !aligned16(out.codes) || (reinterpret_cast<uintptr_t>(out.sf) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(out.gscale) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  // the per-tensor factor a GEMM applies: 1, or 1/sqrt(32) per transformed operand
  // (x H)(w H)^T = 32 x w^T
  const float g = (flags & MXFP4_HADAMARD32) ? 0.17677669529663689f : 1.0f;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t threads = rows_pad * (cols / 32);
  // 256-bit loads when every row of x starts on a 32-byte boundary; one wave of CTAs at the
  // occupancy the runtime reports, walking the blocks with the grid's stride
  const bool v8 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (ldx % 16) == 0;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    int& per_sm = info->mx_ctas_per_sm[v8 ? 1 : 0];
    if (per_sm == 0) {
      int n = 0;
      const cudaError_t e = v8 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::mx_quantize_kernel<true>, 256, 0)
                               : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::mx_quantize_kernel<false>, 256, 0);
      if (e != cudaSuccess || n < 1) return NVFP4_ERR_CUDA;
      per_sm = n;
    }
  }
  int64_t grid = (threads + 255) / 256;
  const int64_t full = static_cast<int64_t>(info->mx_ctas_per_sm[v8 ? 1 : 0]) * info->sm_count;
  if (grid > full) grid = full;
  const int had = (flags & MXFP4_HADAMARD32) ? 1 : 0, inter = (flags & NVFP4_SWIGLU_INTERLEAVE) ? 1 : 0;
  if (v8) {
    nvfp4::mx_quantize_kernel<true><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, cols, ldx, had, inter, static_cast<uint8_t*>(out.codes),
        static_cast<uint8_t*>(out.sf), out.gscale, g);
  } else {
    nvfp4::mx_quantize_kernel<false><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, cols, ldx, had, inter, static_cast<uint8_t*>(out.codes),
        static_cast<uint8_t*>(out.sf), out.gscale, g);
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

NVFP4_API nvfp4_status gemm_mxfp4_pointwise(nvfp4_tensor A, nvfp4_tensor B, const float* bias, int act,
                                            int out_dtype, void* D, int64_t ldd, cudaStream_t stream) {
  if (D == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_RELU) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F16 && out_dtype != NVFP4_OUT_F32)
    return NVFP4_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return NVFP4_ERR_MISALIGNED;
  nvfp4::GemmArgs args{};
  args.bias = bias;
  args.act = act;
  args.out_kind = out_dtype;
  return run_gemm<nvfp4::EPI_POINTWISE, true>(A, B, D, ldd, B.rows, args, stream);
}

NVFP4_API nvfp4_status gemm_mxfp4_plain(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd, cudaStream_t stream) {
  return gemm_mxfp4_pointwise(A, B, nullptr, NVFP4_ACT_NONE, NVFP4_OUT_BF16, D, ldd, stream);
}

template <bool MX>
static nvfp4_status rmsnorm_entry(nvfp4_tensor A, nvfp4_tensor B, const float* w, int head_dim, int64_t n_norm_cols,
                                  float eps, void* D, int64_t ldd, cudaStream_t stream) {
  if (D == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (head_dim != 128 && head_dim != 256) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n_norm_cols < 0 || n_norm_cols > B.rows || n_norm_cols % head_dim != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (n_norm_cols > 0 && w == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (w != nullptr && !aligned16(w)) return NVFP4_ERR_MISALIGNED;
  if (!(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  nvfp4::GemmArgs args{};
  args.w = w;
  args.head_dim = head_dim;
  args.n_norm_cols = static_cast<int>(n_norm_cols);
  args.eps = eps;
  return run_gemm<nvfp4::EPI_RMSNORM, MX>(A, B, D, ldd, B.rows, args, stream);
}

NVFP4_API nvfp4_status gemm_nvfp4_rmsnorm(nvfp4_tensor A, nvfp4_tensor B, const float* w, int head_dim,
                                          int64_t n_norm_cols, float eps, void* D, int64_t ldd,
                                          cudaStream_t stream) {
  return rmsnorm_entry<false>(A, B, w, head_dim, n_norm_cols, eps, D, ldd, stream);
}

NVFP4_API nvfp4_status gemm_mxfp4_rmsnorm(nvfp4_tensor A, nvfp4_tensor B, const float* w, int head_dim,
                                          int64_t n_norm_cols, float eps, void* D, int64_t ldd,
                                          cudaStream_t stream) {
  return rmsnorm_entry<true>(A, B, w, head_dim, n_norm_cols, eps, D, ldd, stream);
}

template <bool MX>
static nvfp4_status swiglu_entry(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd, const nvfp4_tensor* Dq,
                                 cudaStream_t stream) {
  if (D == nullptr && Dq == nullptr) return NVFP4_ERR_INVALID_ARG;
  const int64_t nh = B.rows / 2;
  nvfp4::GemmArgs args{};
  if (Dq != nullptr) {
    if (Dq->codes == nullptr || Dq->sf == nullptr || Dq->gscale == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (Dq->rows != A.rows || Dq->cols != nh) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(Dq->codes) || !aligned16(Dq->sf)) return NVFP4_ERR_MISALIGNED;
    args.q_codes = static_cast<uint8_t*>(Dq->codes);
    args.q_sf = static_cast<uint8_t*>(Dq->sf);
    args.q_gscale = Dq->gscale;
    args.q_cols = static_cast<int>(nh);
  }
  return run_gemm<nvfp4::EPI_SWIGLU, MX>(A, B, D, ldd, nh, args, stream);
}

NVFP4_API nvfp4_status gemm_nvfp4_swiglu(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                                         const nvfp4_tensor* Dq, cudaStream_t stream) {
  return swiglu_entry<false>(A, B, D, ldd, Dq, stream);
}

NVFP4_API nvfp4_status gemm_mxfp4_swiglu(nvfp4_tensor A, nvfp4_tensor B, void* D, int64_t ldd,
                                         const nvfp4_tensor* Dq, cudaStream_t stream) {
  return swiglu_entry<true>(A, B, D, ldd, Dq, stream);
}

NVFP4_API nvfp4_status rmsnorm_heads_bf16(const void* x, int64_t rows, int64_t ldx, const float* w, int head_dim,
                                          int64_t n_norm_cols, float eps, void* y, int64_t ldy,
                                          cudaStream_t stream) {
  if (x == nullptr || y == nullptr || w == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (head_dim != 128 && head_dim != 256) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows <= 0 || n_norm_cols <= 0 || n_norm_cols % head_dim != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ldx < n_norm_cols || ldy < n_norm_cols) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(w) || ldx % 8 || ldy % 8) return NVFP4_ERR_MISALIGNED;
  if (!(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  const int64_t warps = rows * (n_norm_cols / head_dim);
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (head_dim == 256)
    nvfp4::rmsnorm_heads_kernel<256><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, ldx, w, n_norm_cols, eps, static_cast<uint16_t*>(y), ldy);
  else
    nvfp4::rmsnorm_heads_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, ldx, w, n_norm_cols, eps, static_cast<uint16_t*>(y), ldy);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

NVFP4_API nvfp4_status swiglu_bf16(const void* c, int64_t rows, int64_t nh, int64_t ldc, void* y, int64_t ldy,
                                   cudaStream_t stream) {
  if (c == nullptr || y == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || nh <= 0 || nh % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (ldc < 2 * nh || ldy < nh) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(c) || !aligned16(y) || ldc % 8 || ldy % 8) return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  const int64_t threads = rows * (nh / 8);
  const int64_t blocks = (threads + 255) / 256;
  nvfp4::swiglu_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(c), rows, nh, ldc, static_cast<uint16_t*>(y), ldy);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

NVFP4_API const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0)";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel ran out";
  }
  return "unknown status";
}

NVFP4_API int nvfp4_read_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, nvfp4::g_device_status, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyToSymbol(nvfp4::g_device_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

NVFP4_API nvfp4_status nvfp4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1 || limit_ns > 1000000000ll) return NVFP4_ERR_INVALID_ARG;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  nvfp4::selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_ns));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

NVFP4_API int64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

// -------------------------------------------------------------------------------------
// Stream-ordered barrier over peer-mapped signal words (one process per GPU), for the
// row-parallel GEMM whose epilogue adds into the other ranks' output blocks.
// -------------------------------------------------------------------------------------
namespace {

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Thread q < world publishes `epoch` in slot [rank] of rank q's signal words (after a
// system-scope fence, so everything this GPU wrote before, the previous kernels' additions
// into peer blocks included, is visible to q first), then waits until slot [q] of this
// rank's words has reached `epoch`. A wait that runs past limit_ns records
// NVFP4_ERR_DEVICE_TIMEOUT in the device status word and returns.
__global__ void __launch_bounds__(64) signal_barrier_kernel(uint32_t* const* __restrict__ signals, int world,
                                                            int rank, uint32_t epoch, uint64_t limit_ns) {
  const int q = threadIdx.x;
  if (q < world) {
    __threadfence_system();
    st_release_sys(signals[q] + rank, epoch);
  }
  __syncthreads();
  if (q < world) {
    const uint32_t* mine = signals[rank] + q;
    const uint64_t t0 = nvfp4::globaltimer_ns();
    while (static_cast<int32_t>(ld_acquire_sys(mine) - epoch) < 0) {
      if (nvfp4::globaltimer_ns() - t0 > limit_ns) {
        nvfp4::record_status(NVFP4_ERR_DEVICE_TIMEOUT, 70);
        break;
      }
      __nanosleep(64);
    }
  }
}

}  // namespace

NVFP4_API nvfp4_status nvfp4_signal_barrier(uint32_t* const* signals, int world, int rank, uint32_t epoch,
                                            int64_t limit_ns, cudaStream_t stream) {
  if (signals == nullptr || epoch == 0) return NVFP4_ERR_INVALID_ARG;
  if (world < 1 || world > 64 || rank < 0 || rank >= world) return NVFP4_ERR_INVALID_ARG;
  if (limit_ns < 1 || limit_ns > 60000000000ll) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(signals) & 7u) != 0) return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  signal_barrier_kernel<<<1, 64, 0, stream>>>(signals, world, rank, epoch, static_cast<uint64_t>(limit_ns));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

// -------------------------------------------------------------------------------------
// Allocation-free quantiser: nvfp4_quantize with compute_amax = 1, whose scratch (one
// partial maximum per block of 16384 input values, then the tensor's amax) lives in a
// file-scope device array instead of a caller workspace.
// -------------------------------------------------------------------------------------
namespace {

constexpr int kNoAllocPartials = 16384;                     // partial maxima the array holds
constexpr int64_t kNoAllocUnitsPerBlock = 256 * 8;          // 16-byte units per partial (16384 values)
constexpr int64_t kNoAllocMaxValues = static_cast<int64_t>(kNoAllocPartials) * kNoAllocUnitsPerBlock * 8;
static_assert(kNoAllocMaxValues == NVFP4_NOALLOC_MAX_VALUES, "limit stated in the header");

// [0, kNoAllocPartials): partial maxima; [kNoAllocPartials]: the tensor's amax (float bits).
// Every GPU that loads the library holds these 64 KB until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocPartials + 64];

float* g_noalloc_ptr[kMaxDevices] = {nullptr};

// One partial maximum of |x| per block: block b covers 16-byte units
// [b * 2048, (b + 1) * 2048) of the row-major rows x cols view. Written, not accumulated.
__global__ void __launch_bounds__(256) noalloc_amax_partial_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                   int64_t cols, int64_t ldx,
                                                                   float* __restrict__ partials) {
  const int64_t upr = cols >> 3;
  const int64_t total = rows * upr;
  const int64_t base = blockIdx.x * kNoAllocUnitsPerBlock;
  float m = 0.0f;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t u = base + i * 256 + threadIdx.x;
    if (u < total) {
      const int64_t r = u / upr, c = u - r * upr;
      v[i] = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + c * 8));
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w[4] = {v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu, v[i].z & 0x7FFF7FFFu, v[i].w & 0x7FFF7FFFu};
#pragma unroll
    for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(nvfp4::bf16_lo(w[k]), nvfp4::bf16_hi(w[k])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int i = 0; i < 8; ++i) b = fmaxf(b, wmax[i]);
    partials[blockIdx.x] = b;
  }
}

// Maximum of the n partials, written as float bits to *amax_bits.
__global__ void __launch_bounds__(256) noalloc_amax_reduce_kernel(const float* __restrict__ partials, int n,
                                                                  unsigned int* __restrict__ amax_bits) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += 256) m = fmaxf(m, partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int i = 0; i < 8; ++i) b = fmaxf(b, wmax[i]);
    *amax_bits = __float_as_uint(b);
  }
}

// Device address of the scratch array on device `dev` (looked up once per device, with
// that device current).
nvfp4_status noalloc_scratch(int dev, float** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return NVFP4_OK;
}

}  // namespace

NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ldx, int flags,
                                              nvfp4_tensor out, cudaStream_t stream) {
  if (x == nullptr || out.codes == nullptr || out.sf == nullptr || out.gscale == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (flags & ~NVFP4_SWIGLU_INTERLEAVE) return NVFP4_ERR_INVALID_ARG;
  if (out.rows != rows || out.cols != cols) return NVFP4_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || cols % 64 != 0 || ldx < cols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((flags & NVFP4_SWIGLU_INTERLEAVE) && (rows % 2) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // the scratch array holds one partial maximum per 16384 values
  if (rows > kNoAllocMaxValues / cols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || (ldx % 8) != 0 || !aligned16(out.codes) || (reinterpret_cast<uintptr_t>(out.sf) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  int dev;
  DeviceInfo* info;
  nvfp4_status st;
  if ((st = current_device(&dev, &info)) != NVFP4_OK) return st;
  float* scratch;
  if ((st = noalloc_scratch(dev, &scratch)) != NVFP4_OK) return st;

  const uint16_t* xp = static_cast<const uint16_t*>(x);
  const int64_t units = rows * (cols / 8);
  const int blocks = static_cast<int>((units + kNoAllocUnitsPerBlock - 1) / kNoAllocUnitsPerBlock);
  unsigned int* amax_bits = reinterpret_cast<unsigned int*>(scratch + kNoAllocPartials);
  noalloc_amax_partial_kernel<<<blocks, 256, 0, stream>>>(xp, rows, cols, ldx, scratch);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if ((st = launch_status()) != NVFP4_OK) return st;
  noalloc_amax_reduce_kernel<<<1, 256, 0, stream>>>(scratch, blocks, amax_bits);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if ((st = launch_status()) != NVFP4_OK) return st;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t threads = rows_pad * (cols / 64);
  nvfp4::quantize_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      xp, rows, cols, ldx, (flags & NVFP4_SWIGLU_INTERLEAVE) ? 1 : 0, amax_bits, out.gscale,
      static_cast<uint8_t*>(out.codes), static_cast<uint8_t*>(out.sf));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}
