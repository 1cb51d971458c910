"""Shared helpers of the GPU parity tests: move seeded inputs to the device, run the
library through its C ABI, read NVFP4 results back with the oracle's layout decoder,
and the tolerance rule used for bf16 outputs."""
from __future__ import annotations

import numpy as np
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o

# Tolerance for bf16 outputs: per element |g - o| / max(|o|, 1e-2 * rms(o)) <= 2e-2,
# rms over the compared tensor (max relative error 2e-2 with a floor for near-zero
# outputs, so an output that is tiny next to its neighbours is judged on absolute size).
REL_TOL = 2e-2
FLOOR = 1e-2


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    return np.abs(gpu - ref) / np.maximum(np.abs(ref), FLOOR * rms)


def assert_close(gpu, ref, what=""):
    e = rel_err(gpu, ref)
    worst = float(e.max()) if e.size else 0.0
    normwise = float(np.linalg.norm(np.asarray(gpu, np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))
    assert worst <= REL_TOL, f"{what}: max rel err {worst:.3e} (normwise {normwise:.2e}), " \
                             f"{int((e > REL_TOL).sum())} of {e.size} over {REL_TOL}"
    return worst, normwise


def device():
    return torch.device("cuda", 0)


def quantize_gpu(x_bf16: torch.Tensor, interleave=False, G=None) -> ep.NVFP4Tensor:
    """Run the library quantiser on a CPU bf16 tensor (copied to the GPU)."""
    x = x_bf16.to(device())
    t = ep.NVFP4Tensor.empty(x.shape[0], x.shape[1], device())
    if G is not None:
        t.gscale.fill_(float(G))
    ep.nvfp4_quantize(x, t, compute_amax=G is None, interleave=interleave)
    return t


def read_nvfp4(t: ep.NVFP4Tensor):
    """(codes (rows, cols), scales (rows, cols/16), G, raw scale buffer) from the GPU."""
    torch.cuda.synchronize()
    codes = o.unpack_codes(t.codes.cpu().numpy())
    buf = t.sf.cpu().numpy()
    scales = o.unpack_scales(buf, t.rows, t.cols)
    return codes, scales, np.float32(t.gscale.cpu().item()), buf


def nvfp4_from_arrays(codes: np.ndarray, scales: np.ndarray, G: float) -> ep.NVFP4Tensor:
    """Upload codes / scale codes built on the host (oracle layout encoder) to the GPU."""
    rows, cols = codes.shape
    t = ep.NVFP4Tensor.empty(rows, cols, device())
    t.codes.copy_(torch.from_numpy(o.pack_codes(codes)))
    t.sf.copy_(torch.from_numpy(o.pack_scales(scales, cols)))
    t.gscale.fill_(float(G))
    return t


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)
