"""NVFP4 block-scaled GEMM with fused RMSNorm / SwiGLU (+ NVFP4 re-quantisation)
epilogues for B200 (sm_100a), exposed through the C ABI of libnvfp4epi.so.

The Python names mirror the C entry points of include/nvfp4epi.h.
"""
from ._lib import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    FakeQuantizeSTE,
    NVFP4Tensor,
    gemm_mxfp4_plain,
    gemm_mxfp4_pointwise,
    gemm_mxfp4_rmsnorm,
    gemm_mxfp4_swiglu,
    gemm_nvfp4_plain,
    gemm_nvfp4_pointwise,
    gemm_nvfp4_reduce_rows_f32,
    gemm_nvfp4_rmsnorm,
    gemm_nvfp4_swiglu,
    launch_count,
    mxfp4_quantize,
    load,
    nvfp4_fake_quantize,
    nvfp4_quantize,
    nvfp4_quantize_noalloc,
    quantize_workspace_bytes,
    read_device_status,
    rmsnorm_heads_bf16,
    selftest_bounded_wait,
    sf_bytes,
    signal_barrier,
    swiglu_bf16,
)
