"""TPLayer on one GPU (no process group: world size 1) computes exactly what the
unsharded kernels do: the shard packing with the whole weights' scales, the QKV shard's
normalised-column count and both row-parallel down paths (f32 partials for an NCCL
reduce-scatter, and the reduction fused into the GEMM's epilogue). Its outputs are also
checked against the oracle's layer: QKV with per-head RMSNorm, and the FFN chain (SwiGLU,
static re-quantisation, down projection) in float64."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from epilogues_nvfp4_quantize_b200.parallel import TPLayer
import workloads as wk
from oracle import nvfp4_oracle as o
from gpu_util import assert_close, assert_close_chain, device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,reduce", [(256, "nccl"), (384, "nccl"), (256, "fused"), (384, "fused")])
def test_tp_layer_world1_equals_the_unsharded_kernels(M, reduce):
    dev = device()
    heads, hd, K, nh = 4, 128, 512, 512
    x = wk.activations(M, K, 1, seed=M).to(dev)
    wq = wk.weights(3 * heads * hd, K, 1 / np.sqrt(K), seed=1).to(dev)
    wu = wk.weights(2 * nh, K, 1 / np.sqrt(K), seed=2).to(dev)
    wd = wk.weights(K, nh, 1 / np.sqrt(nh), seed=3).to(dev)
    wn_q = torch.from_numpy(wk.norm_weight(hd, 0, 3)).to(dev)
    wn_k = torch.from_numpy(wk.norm_weight(hd, 0, 5)).to(dev)
    T = ep.NVFP4Tensor
    xq = ep.nvfp4_quantize(x, T.empty(M, K, dev))
    G_h = 0.01
    layer = TPLayer(wq, wu, wd, wn_q, wn_k, heads, hd, G_h, reduce=reduce)
    qkv, out = layer.step(xq)
    qkv, out = layer.step(xq)  # a second step reuses (and re-zeroes) the fused output block

    Wq = ep.nvfp4_quantize(wq, T.empty(wq.shape[0], K, dev))
    Wu = ep.nvfp4_quantize(wu, T.empty(wu.shape[0], K, dev), interleave=True)
    Wd = ep.nvfp4_quantize(wd, T.empty(K, nh, dev))
    w_norm = torch.cat([wn_q.repeat(heads), wn_k.repeat(heads)]).float().contiguous()
    qkv_ref = torch.empty_like(qkv)
    ep.gemm_nvfp4_rmsnorm(xq, Wq, w_norm, hd, 2 * heads * hd, 1e-6, qkv_ref)
    h = T.empty(M, nh, dev)
    h.gscale.fill_(G_h)
    ep.gemm_nvfp4_swiglu(xq, Wu, None, h)
    out_ref = torch.empty(M, K, dtype=torch.float32, device=dev)
    ep.gemm_nvfp4_pointwise(h, Wd, out_ref)
    assert torch.equal(qkv, qkv_ref)
    assert torch.equal(out, out_ref)
    assert ep.read_device_status() == 0

    # the oracle's layer on the same inputs
    xc, wqc, wuc, wdc = x.cpu(), wq.cpu(), wu.cpu(), wd.cpu()
    w_norm_np = w_norm.cpu().numpy()
    qkv_o = o.problem_rmsnorm(xc, wqc, w_norm_np, hd, 2 * heads * hd, 1e-6)
    assert_close(qkv.float().cpu().numpy().astype(np.float64), qkv_o, "TPLayer QKV vs oracle")
    h_o = o.problem_swiglu(xc, wuc)
    qh, sh, _ = o.requantize(h_o, np.float32(G_h))
    qd, sd, gd = o.quantized_operand(wdc)
    out_o = o.gemm(o.dequantize(qh, sh, np.float32(G_h)), o.dequantize(qd, sd, gd))
    assert_close_chain(out.cpu().numpy().astype(np.float64), out_o, "TPLayer FFN vs oracle")


def test_tp_layer_bf16_partials_world1_matches_the_oracle():
    dev = device()
    M, heads, hd, K, nh = 256, 4, 128, 512, 512
    x = wk.activations(M, K, 1, seed=9).to(dev)
    wq = wk.weights(3 * heads * hd, K, 1 / np.sqrt(K), seed=1).to(dev)
    wu = wk.weights(2 * nh, K, 1 / np.sqrt(K), seed=2).to(dev)
    wd = wk.weights(K, nh, 1 / np.sqrt(nh), seed=3).to(dev)
    wn = torch.from_numpy(wk.norm_weight(hd, 0, 3)).to(dev)
    xq = ep.nvfp4_quantize(x, ep.NVFP4Tensor.empty(M, K, dev))
    G_h = 0.01
    layer = TPLayer(wq, wu, wd, wn, wn, heads, hd, G_h, reduce="nccl", partials="bf16")
    _, out = layer.step(xq)
    assert out.dtype == torch.bfloat16
    h_o = o.problem_swiglu(x.cpu(), wu.cpu())
    qh, sh, _ = o.requantize(h_o, np.float32(G_h))
    qd, sd, gd = o.quantized_operand(wd.cpu())
    out_o = o.bf16_round(o.gemm(o.dequantize(qh, sh, np.float32(G_h)), o.dequantize(qd, sd, gd)))
    assert_close_chain(out.float().cpu().numpy().astype(np.float64), out_o, "TPLayer bf16 partials vs oracle")


def test_signal_barrier_passes_alone_and_times_out_into_a_status():
    """World size 1: the barrier waits only for its own word and passes. Then a two-rank
    barrier whose second rank does not exist: this rank's wait on a word that nothing sets
    runs out after 2 ms, records NVFP4_ERR_DEVICE_TIMEOUT and returns; the context stays
    usable."""
    dev = device()
    assert ep.read_device_status() == 0
    own = torch.zeros(2, dtype=torch.int32, device=dev)
    ep.signal_barrier(torch.tensor([own.data_ptr()], dtype=torch.int64, device=dev), 0, 1)
    assert ep.read_device_status() == 0
    assert own[0].item() == 1
    other = torch.zeros(2, dtype=torch.int32, device=dev)
    ptrs = torch.tensor([own.data_ptr(), other.data_ptr()], dtype=torch.int64, device=dev)
    ep.signal_barrier(ptrs, 0, 2, limit_ns=2_000_000)
    assert ep.read_device_status() == 6
    assert own[0].item() == 2 and other[0].item() == 2 and own[1].item() == 0
    assert ep.read_device_status() == 0
