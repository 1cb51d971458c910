"""GPU parity of nvfp4_fake_quantize (quantise-dequantise for quantization-aware
distillation) against the oracle: equal to the plain definition except at its ties (a
code or scale tie, or a dequantised value on a bf16 rounding midpoint), and bit for bit
equal to the oracle's float32 evaluation order; and of its straight-through gradient."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import device, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


def _bits(y_bf16_dev):
    return y_bf16_dev.cpu().view(torch.int16).numpy().astype(np.uint16)


def _check(y_bits, x, G):
    """bf16 bits of the GPU result against both statements of the oracle."""
    y_ref, _ = o.fake_quantize(x, G)
    ties = o.fake_quantize_ties(x, G)
    diff = y_bits != o.bf16_bits(y_ref)
    assert not (diff & ~ties).any(), f"{int((diff & ~ties).sum())} values differ outside a tie"
    y32, _ = o.fake_quantize_fp32_order(x, G)
    assert np.array_equal(y_bits, o.bf16_bits(y32))


@pytest.mark.parametrize("rows,cols,outliers", [(256, 1024, 8), (130, 192, 1), (1, 64, 0), (4096, 3072, 3)])
def test_fake_quantize_matches_oracle_bitwise(rows, cols, outliers):
    x = wk.activations(rows, cols, outliers, seed=3 * rows + cols)
    y, g = ep.nvfp4_fake_quantize(x.to(device()))
    G_ref = o.global_scale(x.float().numpy())
    assert float(g.item()) == float(G_ref)
    _check(_bits(y), x.float().numpy(), G_ref)


def test_fake_quantize_static_scale_and_strided_output():
    x = wk.activations(512, 640, 2, seed=5)
    G = np.float32(np.abs(x.float().numpy()).max() / 2688 / 2)  # half the dynamic scale: saturates
    gs = torch.tensor([float(G)], dtype=torch.float32, device=device())
    big = torch.zeros(512, 768, dtype=torch.bfloat16, device=device())
    y, _ = ep.nvfp4_fake_quantize(x.to(device()), y=big[:, 64:704], gscale=gs, compute_amax=False)
    _check(_bits(y.contiguous()), x.float().numpy(), G)
    assert not big[:, :64].any() and not big[:, 704:].any()


def test_fake_quantize_equals_dequantised_nvfp4_quantize():
    # the library's own codes and scales, decoded on the host, give the same bf16 values
    x = wk.activations(384, 512, 2, seed=13)
    q, s, G, _ = read_nvfp4(quantize_gpu(x))
    ls = o.dequantize(q, s, 1.0).astype(np.float32)  # level * scale, exact in fp32
    expect = o.bf16_round((ls * np.float32(G)).astype(np.float64))
    y, _ = ep.nvfp4_fake_quantize(x.to(device()))
    assert np.array_equal(_bits(y), o.bf16_bits(expect))


def test_straight_through_gradient_is_identity():
    x = wk.activations(256, 256, 1, seed=17).to(device()).requires_grad_(True)
    w = torch.randn(256, 256, device=device()).to(torch.bfloat16)
    y = ep.FakeQuantizeSTE.apply(x)
    y_ref, _ = ep.nvfp4_fake_quantize(x.detach())
    assert torch.equal(y, y_ref)
    (y * w).sum().backward()
    assert torch.equal(x.grad, w)
    assert ep.read_device_status() == 0
