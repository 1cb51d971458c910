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


def assert_close_chain(gpu, ref, what="", abs_floor=2e-2, normwise_tol=1e-3):
    """Tolerance for an output computed from re-quantised activations (the down projection
    of the FFN chain): the re-quantisation's codes may legitimately differ from the
    oracle's where the bf16 inputs differ (the quantised-output rule), and each such code
    moves a whole row of the next GEMM's output by about a thousandth of its rms. Per
    element |g - o| <= 2e-2 |o| + 2e-2 rms(o); for the whole output normwise <= 1e-3."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    bound = REL_TOL * np.abs(ref) + abs_floor * rms
    over = np.abs(gpu - ref) > bound
    normwise = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))
    assert not over.any(), f"{what}: {int(over.sum())} of {ref.size} elements over 2e-2|o| + {abs_floor} rms"
    assert normwise <= normwise_tol, f"{what}: normwise {normwise:.2e} over {normwise_tol}"
    return normwise


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


# ---- quantised results against the oracle's plain definition --------------------------
# The GPU takes each rounding decision on float32 quotients (a reciprocal times x); the
# oracle's plain definition decides on the exact quotient. The two may differ only where
# that quotient lies within the oracle's tie band (TIE_REL) of a rounding midpoint; there
# both neighbouring results are correct.

def level_index(codes) -> np.ndarray:
    """Signed E2M1 level index (-7..7; both zeros are 0): adjacent levels differ by 1."""
    c = np.asarray(codes).astype(np.int64)
    return np.where(c & 8, -1, 1) * (c & 7)


def assert_nvfp4_plain(q, s, x, G, what=""):
    """GPU codes q (rows, cols) and scale codes s (rows, cols/16) of the float32 tensor x
    quantised with per-tensor scale G, against the oracle's plain definition:
      - a block scale may differ only where amax_b / (6 G) is a tie, and then by one code;
      - where the scale agrees, a code may differ only at an element tie, by one level;
      - where the scale took the other side of its tie, the codes must be the plain
        rounding of x under the GPU's scale (again up to element ties).
    Returns the numbers of tie-exempted scales and codes."""
    q_ref, s_ref, _ = o.quantize(x, G)
    bt, et = o.quantize_ties(x, G)
    sd = s != s_ref
    assert not (sd & ~bt).any(), f"{what}: {int((sd & ~bt).sum())} block scales differ outside a tie"
    assert np.all(np.abs(s.astype(np.int64) - s_ref.astype(np.int64))[sd] <= 1), f"{what}: scale off by >1"
    same = np.repeat(~sd, 16, axis=1)
    cd = (q != q_ref) & same
    assert not (cd & ~et).any(), f"{what}: {int((cd & ~et).sum())} codes differ outside a tie"
    assert np.all(np.abs(level_index(q) - level_index(q_ref))[cd] <= 1), f"{what}: code off by >1 level"
    alt = 0
    if sd.any():
        q_alt = o.codes_for_scales(x, s, G)
        et_alt = o.code_ties_for_scales(x, s, G)
        ad = (q != q_alt) & ~same
        assert not (ad & ~et_alt).any(), f"{what}: codes under a tie scale differ outside a tie"
        alt = int(ad.sum())
    return int(sd.sum()), int(cd.sum()) + alt


def assert_requant_point13(q, s, got_bf16, ref_bf16, G, what=""):
    """Re-quantised output codes/scales q, s of a fused epilogue whose bf16 output is
    got_bf16, against the oracle re-quantising its own bf16 output ref_bf16 with the same
    static G (reading 13 of the quantised-output comparison):
      - the GPU's codes are the plain quantisation of its own bf16 values (up to ties);
      - in blocks whose bf16 values agree with the oracle's, codes and scales match the
        oracle's (up to ties);
      - everywhere a scale differs from the oracle's by at most one code, and in blocks with
        the oracle's scale a code by at most one level.
    Returns the share of codes that differ from the oracle's."""
    got32 = np.asarray(got_bf16, np.float64).astype(np.float32)
    assert_nvfp4_plain(q, s, got32, G, what + " (vs quantisation of its own bf16 output)")
    q_ref, s_ref, _ = o.requantize(ref_bf16, G)
    rows, cols = q.shape
    blk_same = (np.asarray(got_bf16) == np.asarray(ref_bf16)).reshape(rows, cols // 16, 16).all(axis=2)
    bt, et = o.quantize_ties(np.asarray(ref_bf16, np.float64).astype(np.float32), G)
    sd = s != s_ref
    assert not (sd & blk_same & ~bt).any(), f"{what}: scale differs in a block whose bf16 values agree"
    assert np.all(np.abs(s.astype(np.int64) - s_ref.astype(np.int64)) <= 1), f"{what}: scale off by >1"
    same_scale = np.repeat(~sd, 16, axis=1)
    cd = q != q_ref
    assert not (cd & np.repeat(blk_same, 16, axis=1) & same_scale & ~et).any(), \
        f"{what}: code differs in a block whose bf16 values agree"
    assert np.all(np.abs(level_index(q) - level_index(q_ref))[cd & same_scale] <= 1), \
        f"{what}: code off by more than one level"
    return float(cd.mean())
