"""The layer step (quantiser with its amax pass and grid barrier, the three fused GEMMs)
is capturable in a CUDA graph: a replay reproduces the eager outputs bit for bit. Small
token counts are launch-bound, where a graph removes the per-launch host cost."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
import workloads as wk
from gpu_util import device

pytestmark = pytest.mark.gpu


def test_layer_step_replays_from_a_cuda_graph():
    dev = device()
    M, K, N_qkv, hd, n_norm, nh = 512, 1024, 1536, 256, 1024, 1024
    T = ep.NVFP4Tensor
    x = wk.activations(M, K, 2, seed=1).to(dev)
    Wq = ep.nvfp4_quantize(wk.weights(N_qkv, K, 1 / np.sqrt(K), seed=2).to(dev), T.empty(N_qkv, K, dev))
    Wu = ep.nvfp4_quantize(wk.weights(2 * nh, K, 1 / np.sqrt(K), seed=3).to(dev), T.empty(2 * nh, K, dev),
                           interleave=True)
    Wd = ep.nvfp4_quantize(wk.weights(K, nh, 1 / np.sqrt(nh), seed=4).to(dev), T.empty(K, nh, dev))
    w = torch.from_numpy(np.tile(wk.norm_weight(hd, 0, 3), n_norm // hd)).to(dev)
    ws = torch.empty(ep.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    xq = T.empty(M, K, dev)
    h = T.empty(M, nh, dev)
    h.gscale.fill_(0.005)
    qkv = torch.empty(M, N_qkv, dtype=torch.bfloat16, device=dev)
    out = torch.empty(M, K, dtype=torch.bfloat16, device=dev)

    def step():
        ep.nvfp4_quantize(x, xq, workspace=ws)
        ep.gemm_nvfp4_rmsnorm(xq, Wq, w, hd, n_norm, 1e-6, qkv)
        ep.gemm_nvfp4_swiglu(xq, Wu, None, h)
        ep.gemm_nvfp4_plain(h, Wd, out)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up on the capture stream (attributes, tensor-map encoder)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    qkv_ref, out_ref = qkv.clone(), out.clone()
    qkv.zero_()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(qkv, qkv_ref) and torch.equal(out, out_ref)
    assert ep.read_device_status() == 0
