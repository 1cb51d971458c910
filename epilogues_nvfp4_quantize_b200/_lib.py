"""ctypes binding of libnvfp4epi.so: argument marshalling only.

Every computation runs in the library's CUDA kernels; this module turns torch tensors
into device pointers, sizes and the current stream, and raises RuntimeError on a
non-OK status. There is no CPU fallback: if the shared library is missing or cannot
be loaded, every call fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4epi.so")

SWIGLU_INTERLEAVE = 1

# Entry points declared in include/nvfp4epi.h (kept in sync by tests/test_abi.py).
EXPORTS = (
    "nvfp4_sf_bytes", "nvfp4_quantize_workspace_bytes", "nvfp4_quantize",
    "gemm_nvfp4_plain", "gemm_nvfp4_rmsnorm", "gemm_nvfp4_swiglu",
    "rmsnorm_heads_bf16", "swiglu_bf16", "nvfp4_status_string",
    "nvfp4_read_device_status", "nvfp4_selftest_bounded_wait", "nvfp4_launch_count",
    "nvfp4_quantize_noalloc", "nvfp4_fake_quantize", "gemm_nvfp4_pointwise",
    "mxfp4_sf_bytes", "mxfp4_quantize", "gemm_mxfp4_pointwise", "gemm_mxfp4_plain",
    "gemm_mxfp4_rmsnorm", "gemm_mxfp4_swiglu", "gemm_nvfp4_reduce_rows_f32", "nvfp4_signal_barrier",
)


class _Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("gscale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_lib = None


def load() -> ctypes.CDLL:
    """Load the shared library (once). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libnvfp4epi.so not built at {LIB_PATH}; run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp, i32, f32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "nvfp4_sf_bytes": (i64, [i64, i64]),
        "nvfp4_quantize_workspace_bytes": (i64, []),
        "nvfp4_quantize": (i32, [vp, i64, i64, i64, i32, i32, _Tensor, vp, vp]),
        "gemm_nvfp4_plain": (i32, [_Tensor, _Tensor, vp, i64, vp]),
        "gemm_nvfp4_rmsnorm": (i32, [_Tensor, _Tensor, vp, i32, i64, f32, vp, i64, vp]),
        "gemm_nvfp4_swiglu": (i32, [_Tensor, _Tensor, vp, i64, ctypes.POINTER(_Tensor), vp]),
        "rmsnorm_heads_bf16": (i32, [vp, i64, i64, vp, i32, i64, f32, vp, i64, vp]),
        "swiglu_bf16": (i32, [vp, i64, i64, i64, vp, i64, vp]),
        "nvfp4_status_string": (ctypes.c_char_p, [i32]),
        "nvfp4_read_device_status": (i32, [vp]),
        "nvfp4_selftest_bounded_wait": (i32, [i64, vp]),
        "nvfp4_launch_count": (i64, []),
        "nvfp4_quantize_noalloc": (i32, [vp, i64, i64, i64, i32, _Tensor, vp]),
        "nvfp4_fake_quantize": (i32, [vp, i64, i64, i64, i32, vp, vp, i64, vp, vp]),
        "gemm_nvfp4_pointwise": (i32, [_Tensor, _Tensor, vp, i32, i32, vp, i64, ctypes.POINTER(_Tensor), vp]),
        "gemm_nvfp4_reduce_rows_f32": (i32, [_Tensor, _Tensor, vp, i32, i64, i64, vp]),
        "mxfp4_sf_bytes": (i64, [i64, i64]),
        "mxfp4_quantize": (i32, [vp, i64, i64, i64, i32, _Tensor, vp]),
        "gemm_mxfp4_pointwise": (i32, [_Tensor, _Tensor, vp, i32, i32, vp, i64, vp]),
        "gemm_mxfp4_plain": (i32, [_Tensor, _Tensor, vp, i64, vp]),
        "gemm_mxfp4_rmsnorm": (i32, [_Tensor, _Tensor, vp, i32, i64, f32, vp, i64, vp]),
        "gemm_mxfp4_swiglu": (i32, [_Tensor, _Tensor, vp, i64, ctypes.POINTER(_Tensor), vp]),
        "nvfp4_signal_barrier": (i32, [vp, i32, i32, ctypes.c_uint32, i64, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != 0:
        msg = load().nvfp4_status_string(status).decode()
        raise RuntimeError(f"{what}: {msg} (status {status})")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


class NVFP4Tensor:
    """Device buffers of an NVFP4 tensor (see nvfp4_tensor in include/nvfp4epi.h)."""

    def __init__(self, codes: torch.Tensor, sf: torch.Tensor, gscale: torch.Tensor, rows: int, cols: int):
        self.codes, self.sf, self.gscale, self.rows, self.cols = codes, sf, gscale, rows, cols

    @classmethod
    def empty(cls, rows: int, cols: int, device="cuda") -> "NVFP4Tensor":
        return cls(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                   torch.empty((sf_bytes(rows, cols),), dtype=torch.uint8, device=device),
                   torch.empty((1,), dtype=torch.float32, device=device), rows, cols)

    @classmethod
    def empty_mx(cls, rows: int, cols: int, device="cuda") -> "NVFP4Tensor":
        """Buffers of an MXFP4 tensor (E8M0 scales per 32 values; see mxfp4_quantize)."""
        return cls(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                   torch.empty((int(load().mxfp4_sf_bytes(rows, cols)),), dtype=torch.uint8, device=device),
                   torch.empty((1,), dtype=torch.float32, device=device), rows, cols)

    def c(self) -> _Tensor:
        return _Tensor(self.codes.data_ptr(), self.sf.data_ptr(), self.gscale.data_ptr(), self.rows, self.cols)

    def nbytes(self) -> int:
        return self.codes.numel() + self.sf.numel() + 4


def sf_bytes(rows: int, cols: int) -> int:
    return int(load().nvfp4_sf_bytes(rows, cols))


def quantize_workspace_bytes() -> int:
    return int(load().nvfp4_quantize_workspace_bytes())


def _workspace(workspace: Optional[torch.Tensor], compute_amax: bool, device) -> Optional[torch.Tensor]:
    """The caller's workspace (checked for size), or a new one when none is given."""
    if not compute_amax:
        return workspace
    need = quantize_workspace_bytes()
    if workspace is None:
        return torch.empty((need,), dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace holds {workspace.numel() * workspace.element_size()} bytes, needs {need}")
    return workspace


def nvfp4_quantize(x: torch.Tensor, out: NVFP4Tensor, compute_amax: bool = True, interleave: bool = False,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> NVFP4Tensor:
    """Quantise a bf16 2-D CUDA tensor into `out` (see nvfp4_quantize in the header)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    workspace = _workspace(workspace, compute_amax, x.device)
    _check(load().nvfp4_quantize(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), int(compute_amax),
                                 SWIGLU_INTERLEAVE if interleave else 0, out.c(), _ptr(workspace),
                                 _stream(stream)), "nvfp4_quantize")
    return out


def _out2d(D: Optional[torch.Tensor]):
    if D is None:
        return None, 0
    if D.dtype != torch.bfloat16 or D.dim() != 2 or D.stride(1) != 1:
        raise ValueError("outputs are 2-D bf16 tensors with unit column stride")
    return D.data_ptr(), D.stride(0)


def gemm_nvfp4_plain(A: NVFP4Tensor, B: NVFP4Tensor, D: torch.Tensor, stream=None) -> torch.Tensor:
    p, ld = _out2d(D)
    _check(load().gemm_nvfp4_plain(A.c(), B.c(), p, ld, _stream(stream)), "gemm_nvfp4_plain")
    return D


def gemm_nvfp4_rmsnorm(A: NVFP4Tensor, B: NVFP4Tensor, w: Optional[torch.Tensor], head_dim: int,
                       n_norm_cols: int, eps: float, D: torch.Tensor, stream=None) -> torch.Tensor:
    if w is not None and (w.dtype != torch.float32 or not w.is_contiguous()):
        raise ValueError("w must be a contiguous float32 tensor")
    p, ld = _out2d(D)
    _check(load().gemm_nvfp4_rmsnorm(A.c(), B.c(), _ptr(w), head_dim, n_norm_cols, eps, p, ld, _stream(stream)),
           "gemm_nvfp4_rmsnorm")
    return D


def gemm_nvfp4_swiglu(A: NVFP4Tensor, B: NVFP4Tensor, D: Optional[torch.Tensor] = None,
                      Dq: Optional[NVFP4Tensor] = None, stream=None):
    p, ld = _out2d(D)
    dq = ctypes.pointer(Dq.c()) if Dq is not None else None
    _check(load().gemm_nvfp4_swiglu(A.c(), B.c(), p, ld, dq, _stream(stream)), "gemm_nvfp4_swiglu")
    return D, Dq


ACT_NONE, ACT_RELU = 0, 1
_OUT_KIND = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}


def gemm_nvfp4_pointwise(A: NVFP4Tensor, B: NVFP4Tensor, D: Optional[torch.Tensor] = None,
                         bias: Optional[torch.Tensor] = None, relu: bool = False,
                         Dq: Optional[NVFP4Tensor] = None, stream=None):
    """D = cast(act(G_A G_B acc + bias)) in D's dtype (bf16, f16 or f32) and/or Dq = NVFP4 of
    bf16 of it with Dq's static scale (see gemm_nvfp4_pointwise in the header)."""
    if bias is not None and (bias.dtype != torch.float32 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous float32 tensor")
    if D is not None:
        if D.dtype not in _OUT_KIND or D.dim() != 2 or D.stride(1) != 1:
            raise ValueError("D must be a 2-D bf16, f16 or f32 tensor with unit column stride")
        p, ld, kind = D.data_ptr(), D.stride(0), _OUT_KIND[D.dtype]
    else:
        p, ld, kind = None, 0, 0
    dq = ctypes.pointer(Dq.c()) if Dq is not None else None
    _check(load().gemm_nvfp4_pointwise(A.c(), B.c(), _ptr(bias), ACT_RELU if relu else ACT_NONE, kind, p, ld, dq,
                                       _stream(stream)), "gemm_nvfp4_pointwise")
    return D, Dq


def gemm_nvfp4_reduce_rows_f32(A: NVFP4Tensor, B: NVFP4Tensor, dst_ptrs: torch.Tensor, rows_per_rank: int,
                               ldd: int, stream=None):
    """Add row m of G_A G_B (A B^T) (float32) into destination m // rows_per_rank at row
    m % rows_per_rank (see gemm_nvfp4_reduce_rows_f32 in the header). dst_ptrs: a device
    int64 tensor of the destinations' addresses (float32 blocks with leading dimension ldd)."""
    if dst_ptrs.dtype != torch.int64 or dst_ptrs.dim() != 1 or not dst_ptrs.is_cuda or not dst_ptrs.is_contiguous():
        raise ValueError("dst_ptrs must be a contiguous 1-D int64 tensor on the GPU")
    _check(load().gemm_nvfp4_reduce_rows_f32(A.c(), B.c(), dst_ptrs.data_ptr(), dst_ptrs.numel(), rows_per_rank, ldd,
                                             _stream(stream)), "gemm_nvfp4_reduce_rows_f32")


MXFP4_HADAMARD32 = 2


def mxfp4_quantize(x: torch.Tensor, out: NVFP4Tensor, hadamard: bool = False, interleave: bool = False,
                   stream=None) -> NVFP4Tensor:
    """MXFP4-quantise a bf16 2-D CUDA tensor (optionally after the 32-point block Hadamard
    transform, optionally with the SwiGLU gate/up row interleave) into `out` (from
    NVFP4Tensor.empty_mx); see mxfp4_quantize in the header."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    flags = (MXFP4_HADAMARD32 if hadamard else 0) | (SWIGLU_INTERLEAVE if interleave else 0)
    _check(load().mxfp4_quantize(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), flags, out.c(),
                                 _stream(stream)), "mxfp4_quantize")
    return out


def gemm_mxfp4_rmsnorm(A: NVFP4Tensor, B: NVFP4Tensor, w: Optional[torch.Tensor], head_dim: int,
                       n_norm_cols: int, eps: float, D: torch.Tensor, stream=None) -> torch.Tensor:
    if w is not None and (w.dtype != torch.float32 or not w.is_contiguous()):
        raise ValueError("w must be a contiguous float32 tensor")
    p, ld = _out2d(D)
    _check(load().gemm_mxfp4_rmsnorm(A.c(), B.c(), _ptr(w), head_dim, n_norm_cols, eps, p, ld, _stream(stream)),
           "gemm_mxfp4_rmsnorm")
    return D


def gemm_mxfp4_swiglu(A: NVFP4Tensor, B: NVFP4Tensor, D: Optional[torch.Tensor] = None,
                      Dq: Optional[NVFP4Tensor] = None, stream=None):
    p, ld = _out2d(D)
    dq = ctypes.pointer(Dq.c()) if Dq is not None else None
    _check(load().gemm_mxfp4_swiglu(A.c(), B.c(), p, ld, dq, _stream(stream)), "gemm_mxfp4_swiglu")
    return D, Dq


def gemm_mxfp4_pointwise(A: NVFP4Tensor, B: NVFP4Tensor, D: torch.Tensor, bias: Optional[torch.Tensor] = None,
                         relu: bool = False, stream=None) -> torch.Tensor:
    if bias is not None and (bias.dtype != torch.float32 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous float32 tensor")
    if D.dtype not in _OUT_KIND or D.dim() != 2 or D.stride(1) != 1:
        raise ValueError("D must be a 2-D bf16, f16 or f32 tensor with unit column stride")
    _check(load().gemm_mxfp4_pointwise(A.c(), B.c(), _ptr(bias), ACT_RELU if relu else ACT_NONE, _OUT_KIND[D.dtype],
                                       D.data_ptr(), D.stride(0), _stream(stream)), "gemm_mxfp4_pointwise")
    return D


def gemm_mxfp4_plain(A: NVFP4Tensor, B: NVFP4Tensor, D: torch.Tensor, stream=None) -> torch.Tensor:
    p, ld = _out2d(D)
    _check(load().gemm_mxfp4_plain(A.c(), B.c(), p, ld, _stream(stream)), "gemm_mxfp4_plain")
    return D


def rmsnorm_heads_bf16(x: torch.Tensor, w: torch.Tensor, head_dim: int, n_norm_cols: int, eps: float,
                       y: torch.Tensor, stream=None) -> torch.Tensor:
    px, ldx = _out2d(x)
    py, ldy = _out2d(y)
    _check(load().rmsnorm_heads_bf16(px, x.shape[0], ldx, w.data_ptr(), head_dim, n_norm_cols, eps, py, ldy,
                                     _stream(stream)), "rmsnorm_heads_bf16")
    return y


def swiglu_bf16(c: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
    pc, ldc = _out2d(c)
    py, ldy = _out2d(y)
    _check(load().swiglu_bf16(pc, c.shape[0], c.shape[1] // 2, ldc, py, ldy, _stream(stream)), "swiglu_bf16")
    return y


NOALLOC_MAX_VALUES = 268435456


def nvfp4_quantize_noalloc(x: torch.Tensor, out: NVFP4Tensor, interleave: bool = False, stream=None) -> NVFP4Tensor:
    """nvfp4_quantize with the per-tensor scale derived on the device, for callers that
    cannot allocate device memory: the library keeps the reduction's scratch in its own
    static device memory, so no workspace is needed (see nvfp4_quantize_noalloc in the
    header for the size limit and the rule that overlapping calls race)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    _check(load().nvfp4_quantize_noalloc(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0),
                                         SWIGLU_INTERLEAVE if interleave else 0, out.c(), _stream(stream)),
           "nvfp4_quantize_noalloc")
    return out


def nvfp4_fake_quantize(x: torch.Tensor, y: Optional[torch.Tensor] = None, gscale: Optional[torch.Tensor] = None,
                        compute_amax: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """Quantise-dequantise a 2-D bf16 CUDA tensor through NVFP4 (see nvfp4_fake_quantize in
    the header). Returns (y, gscale); gscale is a 1-element float32 device tensor, written
    when compute_amax, read otherwise."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    if y is None:
        y = torch.empty_like(x, memory_format=torch.contiguous_format)
    py, ldy = _out2d(y)
    if gscale is None:
        if not compute_amax:
            raise ValueError("a static scale needs gscale")
        gscale = torch.empty((1,), dtype=torch.float32, device=x.device)
    workspace = _workspace(workspace, compute_amax, x.device)
    _check(load().nvfp4_fake_quantize(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), int(compute_amax),
                                      gscale.data_ptr(), py, ldy, _ptr(workspace), _stream(stream)),
           "nvfp4_fake_quantize")
    return y, gscale


class FakeQuantizeSTE(torch.autograd.Function):
    """y = nvfp4_fake_quantize(x) forward; identity backward (straight-through estimator:
    the rounding is left out of the gradient, which flows at full precision)."""

    @staticmethod
    def forward(ctx, x, gscale=None, compute_amax=True):
        y, _ = nvfp4_fake_quantize(x.contiguous(), gscale=gscale, compute_amax=compute_amax)
        return y

    @staticmethod
    def backward(ctx, grad_y):
        return grad_y, None, None


def read_device_status(stream=None) -> int:
    return int(load().nvfp4_read_device_status(_stream(stream)))


def signal_barrier(signal_ptrs: torch.Tensor, rank: int, epoch: int, limit_ns: int = 10_000_000_000,
                   stream=None) -> None:
    """Barrier over peer-mapped signal words: signal_ptrs is a device int64 tensor of the
    world's signal-array addresses (see nvfp4_signal_barrier). A rank that does not arrive
    within limit_ns ends this rank's wait with NVFP4_ERR_DEVICE_TIMEOUT in the device status
    word (read_device_status) instead of holding the GPU."""
    if signal_ptrs.dtype != torch.int64 or not signal_ptrs.is_cuda:
        raise RuntimeError("signal_ptrs must be a CUDA int64 tensor of addresses")
    _check(load().nvfp4_signal_barrier(signal_ptrs.data_ptr(), signal_ptrs.numel(), rank, epoch & 0xFFFFFFFF,
                                       limit_ns, _stream(stream)), "nvfp4_signal_barrier")


def selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(load().nvfp4_selftest_bounded_wait(limit_ns, _stream(stream)), "nvfp4_selftest_bounded_wait")


def launch_count() -> int:
    return int(load().nvfp4_launch_count())
