"""GPU parity of nvfp4_quantize against the oracle: codes, block scales and the
per-tensor scale must agree bit for bit (both sides take every decision with the same
IEEE float32 operations)."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import device, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


def _check_bitwise(x_bf16, t, G_static=None, interleave=False):
    x = x_bf16.float().numpy()
    if interleave:
        x = o.interleave_gate_up(x)
    q_ref, s_ref, G_ref = o.quantize(x, G_static)
    q, s, G, buf = read_nvfp4(t)
    assert G == G_ref
    assert np.array_equal(s, s_ref), f"{int((s != s_ref).sum())} scale mismatches"
    assert np.array_equal(q, q_ref), f"{int((q != q_ref).sum())} code mismatches"
    # padding bytes of the scale buffer are zero
    assert np.array_equal(buf, o.pack_scales(s_ref, x.shape[1]))


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


def test_quantize_reuses_workspace_across_calls():
    ws = torch.empty(ep.quantize_workspace_bytes(), dtype=torch.uint8, device=device())
    for seed in (1, 2):
        x = wk.activations(128, 256, 1, seed=seed)
        t = ep.NVFP4Tensor.empty(128, 256, device())
        ep.nvfp4_quantize(x.to(device()), t, workspace=ws)
        _check_bitwise(x, t)
