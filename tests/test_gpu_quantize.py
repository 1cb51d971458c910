"""GPU parity of nvfp4_quantize against the oracle.

- Against the plain definition (exact quotients): the per-tensor scale bit for bit; block
  scales and codes equal except at rounding ties, where they may take the neighbouring
  value (one code, one level).
- Against the oracle's float32 evaluation order (reciprocal times x, the order the kernel
  uses): codes, scales and padding bytes bit for bit."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_nvfp4_plain, device, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


def _check_bitwise(x_bf16, t, G_static=None, interleave=False):
    x = x_bf16.float().numpy()
    if interleave:
        x = o.interleave_gate_up(x)
    q, s, G, buf = read_nvfp4(t)
    G_ref = o.global_scale(x) if G_static is None else np.float32(G_static)
    assert G == G_ref
    assert_nvfp4_plain(q, s, x, G_ref, "nvfp4_quantize")
    q32, s32, _ = o.quantize_fp32_order(x, G_static)
    assert np.array_equal(s, s32), f"{int((s != s32).sum())} scale mismatches (float32 order)"
    assert np.array_equal(q, q32), f"{int((q != q32).sum())} code mismatches (float32 order)"
    # padding bytes of the scale buffer are zero
    assert np.array_equal(buf, o.pack_scales(s32, x.shape[1]))


@pytest.mark.parametrize("rows,cols,outliers", [(256, 1024, 8), (130, 192, 1), (1, 64, 0), (4096, 3072, 3)])
def test_quantize_matches_oracle_bitwise(rows, cols, outliers):
    x = wk.activations(rows, cols, outliers, seed=rows + cols)
    _check_bitwise(x, quantize_gpu(x))


def test_quantize_interleaved_weight():
    w = wk.weights(2 * 384, 512, 1 / np.sqrt(512), seed=7)
    t = quantize_gpu(w, interleave=True)
    _check_bitwise(w, t, interleave=True)


@pytest.mark.parametrize("nh,cols", [(100, 320), (1000, 64)])
def test_quantize_interleaved_ragged(nh, cols):
    # 2*nh rows: the halves start off a 64-row boundary and the last 128-row block is partial
    w = wk.weights(2 * nh, cols, 1 / np.sqrt(cols), seed=nh)
    _check_bitwise(w, quantize_gpu(w, interleave=True), interleave=True)


def test_quantize_static_scale_many_blocks_per_cta():
    x = wk.activations(4000, 1984, 2, seed=21)  # 32 x 8 chunks of 128 rows x 256 columns
    G = np.float32(np.abs(x.float().numpy()).max() / 2688)
    _check_bitwise(x, quantize_gpu(x, G=G), G_static=G)


def test_quantize_static_scale_including_saturation():
    x = wk.activations(256, 512, 2, seed=9)
    G = np.float32(np.abs(x.float().numpy()).max() / 2688 / 4)  # too small: saturates
    _check_bitwise(x, quantize_gpu(x, G=G), G_static=G)
    G2 = np.float32(0.0123)
    _check_bitwise(x, quantize_gpu(x, G=G2), G_static=G2)


def test_quantize_zero_tensor_and_zero_blocks():
    x = torch.zeros(128, 128, dtype=torch.bfloat16)
    t = quantize_gpu(x)
    q, s, G, buf = read_nvfp4(t)
    assert G == 0 and not q.any() and not buf.any()
    y = wk.activations(128, 128, 0, seed=3)
    y[5, 16:48] = 0
    _check_bitwise(y, quantize_gpu(y))


def test_quantize_small_values_round_to_signed_zero():
    # values far below the block's step round to zero with their sign kept
    x = np.zeros((128, 64), np.float32)
    x[:, 0] = 6.0
    x[:, 1] = -0.01
    x[:, 2] = 0.01
    x[:, 3] = -1e-30
    xt = torch.from_numpy(x).to(torch.bfloat16)
    _check_bitwise(xt, quantize_gpu(xt))


def test_quantize_strided_rows():
    big = wk.activations(256, 768, 2, seed=11).to(device())
    view = big[:, 128:640]  # ldx = 768, cols = 512
    t = ep.NVFP4Tensor.empty(256, 512, device())
    ep.nvfp4_quantize(view, t)
    _check_bitwise(big[:, 128:640].cpu().contiguous(), t)


@pytest.mark.parametrize("rows,cols", [(256, 512), (130, 192)])
def test_quantize_contiguous_off_a_32_byte_boundary(rows, cols):
    """A contiguous x that starts 16 bytes past a 32-byte boundary takes the row kernel with
    128-bit accesses; the same values at a 32-byte boundary take the flat kernel. Both match
    the oracle bit for bit."""
    x = wk.activations(rows, cols, 2, seed=rows)
    flat = torch.empty(rows * cols + 8, dtype=torch.bfloat16, device=device())
    view = flat[8:].view(rows, cols)
    assert view.data_ptr() % 32 == 16
    view.copy_(x.to(device()))
    t = ep.NVFP4Tensor.empty(rows, cols, device())
    ep.nvfp4_quantize(view, t)
    _check_bitwise(x, t)
    _check_bitwise(x, quantize_gpu(x))


def test_quantize_reuses_workspace_across_calls():
    ws = torch.empty(ep.quantize_workspace_bytes(), dtype=torch.uint8, device=device())
    for seed in (1, 2):
        x = wk.activations(128, 256, 1, seed=seed)
        t = ep.NVFP4Tensor.empty(128, 256, device())
        ep.nvfp4_quantize(x.to(device()), t, workspace=ws)
        _check_bitwise(x, t)


def test_quantize_ties_follow_the_float32_order_and_stay_within_the_tie_rule():
    """Weights with their dynamic scale: G = amax / (6 * 448) turns many x / d into ratios
    of short bf16 numbers that sit on a rounding midpoint except for the float32 rounding
    of G (and amax_b / (6 G) = 448 * amax_b / amax, a ratio of two bf16 numbers, sits on a
    scale midpoint the same way). For this seed the plain definition and the float32 order
    disagree on about 1 % of the block scales and 0.3 % of the codes. The kernel must take
    the float32 order's side there, inside the tie rule."""
    w = wk.weights(2048, 3072, 1 / np.sqrt(3072), seed=3)
    t = quantize_gpu(w)
    q, s, G, _ = read_nvfp4(t)
    wf = w.float().numpy()
    exempt_scales, exempt_codes = assert_nvfp4_plain(q, s, wf, G, "weights")
    assert exempt_scales > 0 and exempt_codes > 0
    q32, s32, _ = o.quantize_fp32_order(wf)
    assert np.array_equal(q, q32) and np.array_equal(s, s32)
