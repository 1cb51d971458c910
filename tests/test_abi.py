"""The C-ABI library loads, exports every entry point the header declares, and its
host-side argument checks answer without a GPU (no compute call is made here)."""
import ctypes
import os
import re

import numpy as np
import pytest

import epilogues_nvfp4_quantize_b200 as ep
from epilogues_nvfp4_quantize_b200 import _lib
from oracle import nvfp4_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4epi.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from epilogues_nvfp4_quantize_b200.build import build
    build()
    return ep.load()


def test_header_and_binding_agree():
    assert _declared() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_scale_buffer_size_matches_layout(lib):
    for rows, cols in [(1, 64), (128, 256), (130, 192), (4096, 3072), (16384, 12288)]:
        assert ep.sf_bytes(rows, cols) == o.sf_bytes(rows, cols)
    assert lib.nvfp4_sf_bytes(-1, 16) == -1


def test_status_strings(lib):
    for s in range(7):
        assert lib.nvfp4_status_string(s).decode()
    assert b"unknown" in lib.nvfp4_status_string(99)


def _t(rows=128, cols=256, codes=16, sf=16, g=16):
    return _lib._Tensor(codes, sf, g, rows, cols)


def test_argument_checks_return_status_without_gpu(lib):
    INVALID, SHAPE, MISALIGNED = 1, 2, 3
    # quantize: null input, bad flags, shape rules, alignment
    assert lib.nvfp4_quantize(None, 128, 256, 256, 0, 0, _t(), None, None) == INVALID
    assert lib.nvfp4_quantize(16, 128, 256, 256, 0, 4, _t(), None, None) == INVALID
    assert lib.nvfp4_quantize(16, 128, 256, 256, 1, 0, _t(), None, None) == INVALID      # no workspace
    assert lib.nvfp4_quantize(16, 128, 96, 96, 0, 0, _t(cols=96), None, None) == SHAPE   # cols % 64
    assert lib.nvfp4_quantize(16, 3, 64, 64, 0, 1, _t(3, 64), None, None) == SHAPE      # odd rows, interleave
    assert lib.nvfp4_quantize(18, 128, 256, 256, 0, 0, _t(), None, None) == MISALIGNED
    assert lib.nvfp4_quantize(16, 128, 256, 200, 0, 0, _t(), None, None) == SHAPE       # ldx < cols
    # gemm: shape rules
    assert lib.gemm_nvfp4_plain(_t(100, 256), _t(256, 256), 16, 256, None) == SHAPE    # M % 128
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(128, 256), 16, 128, None) == SHAPE    # N % 256
    assert lib.gemm_nvfp4_plain(_t(128, 128), _t(256, 128), 16, 256, None) == SHAPE    # K % 256
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(256, 512), 16, 256, None) == INVALID  # K mismatch
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(256, 256), None, 256, None) == INVALID
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(256, 256), 16, 200, None) == INVALID  # ldd < N
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(256, 256), 24, 256, None) == MISALIGNED
    assert lib.gemm_nvfp4_plain(_t(128, 256, codes=8), _t(256, 256), 16, 256, None) == MISALIGNED
    assert lib.gemm_nvfp4_rmsnorm(_t(), _t(256, 256), 16, 64, 256, 1e-6, 16, 256, None) == SHAPE
    assert lib.gemm_nvfp4_rmsnorm(_t(), _t(256, 256), 16, 256, 128, 1e-6, 16, 256, None) == SHAPE
    assert lib.gemm_nvfp4_rmsnorm(_t(), _t(256, 256), None, 256, 256, 1e-6, 16, 256, None) == INVALID
    assert lib.gemm_nvfp4_swiglu(_t(), _t(256, 256), None, 0, None, None) == INVALID
    bad = _t(128, 64)
    assert lib.gemm_nvfp4_swiglu(_t(), _t(256, 256), None, 0, ctypes.pointer(bad), None) == INVALID
    assert lib.rmsnorm_heads_bf16(16, 4, 256, 16, 256, 100, 1e-6, 16, 256, None) == SHAPE
    assert lib.swiglu_bf16(16, 4, 12, 24, 16, 12, None) == SHAPE
    assert lib.nvfp4_selftest_bounded_wait(0, None) == INVALID
    # row-parallel reduce: destinations array, ranks, rows per rank, pitch
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), None, 2, 128, 256, None) == INVALID
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 12, 2, 128, 256, None) == INVALID  # dst % 8
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 16, 0, 128, 256, None) == INVALID
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 16, 4, 64, 256, None) == SHAPE  # rows % 128
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 16, 1, 128, 256, None) == SHAPE  # M != w*rows
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 16, 2, 128, 200, None) == INVALID  # ldd < N
    assert lib.gemm_nvfp4_reduce_rows_f32(_t(256, 256), _t(256, 256), 16, 2, 128, 258, None) == MISALIGNED
    # signal barrier: pointer array, world, rank, epoch, limit
    assert lib.nvfp4_signal_barrier(None, 2, 0, 1, 1000, None) == INVALID
    assert lib.nvfp4_signal_barrier(16, 0, 0, 1, 1000, None) == INVALID      # world < 1
    assert lib.nvfp4_signal_barrier(16, 2, 2, 1, 1000, None) == INVALID      # rank >= world
    assert lib.nvfp4_signal_barrier(16, 2, 0, 0, 1000, None) == INVALID      # epoch 0
    assert lib.nvfp4_signal_barrier(16, 2, 0, 1, 0, None) == INVALID         # limit 0
    assert lib.nvfp4_signal_barrier(12, 2, 0, 1, 1000, None) == MISALIGNED   # array % 8


def test_empty_inputs_are_rejected_before_any_launch(lib):
    """Zero rows or columns are a shape error on every entry point that takes sizes: the
    kernels never see an empty grid."""
    SHAPE = 2
    assert lib.nvfp4_quantize(16, 0, 256, 256, 0, 0, _t(0, 256), None, None) == SHAPE
    assert lib.nvfp4_quantize(16, 128, 0, 256, 0, 0, _t(128, 0), None, None) == SHAPE
    assert lib.nvfp4_quantize_noalloc(16, 0, 256, 256, 0, _t(0, 256), None) == SHAPE
    assert lib.nvfp4_fake_quantize(16, 0, 256, 256, 0, 16, 16, 256, None, None) == SHAPE
    assert lib.mxfp4_quantize(16, 0, 256, 256, 0, _t(0, 256), None) == SHAPE
    assert lib.gemm_nvfp4_plain(_t(0, 256), _t(256, 256), 16, 256, None) == SHAPE      # M = 0
    assert lib.gemm_nvfp4_plain(_t(128, 256), _t(0, 256), 16, 256, None) == SHAPE      # N = 0
    assert lib.gemm_nvfp4_plain(_t(128, 0), _t(256, 0), 16, 256, None) == SHAPE        # K = 0
    assert lib.gemm_mxfp4_plain(_t(0, 256), _t(256, 256), 16, 256, None) == SHAPE
    assert lib.rmsnorm_heads_bf16(16, 0, 256, 16, 128, 256, 1e-6, 16, 256, None) == SHAPE
    assert lib.swiglu_bf16(16, 0, 16, 32, 16, 16, None) == SHAPE


def test_valid_call_without_a_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # all checks pass, so the library asks the runtime for a device and reports it
    st = lib.nvfp4_quantize(16, 128, 256, 256, 0, 0, _t(), None, None)
    assert st in (4, 5)
    with pytest.raises(RuntimeError):
        _lib._check(st, "nvfp4_quantize")
