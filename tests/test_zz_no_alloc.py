"""The allocation-free quantiser, for callers that cannot allocate device memory (a host
application that owns the whole GPU, or a latency-critical path where cudaMalloc may
synchronise the device): nvfp4_quantize_noalloc keeps the amax reduction's scratch in the
library's own static device memory. Its results must equal those of nvfp4_quantize with a
caller workspace, bit for bit, on consecutive calls (the shared scratch keeps the previous
call's values). This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from epilogues_nvfp4_quantize_b200 import _lib
from oracle import nvfp4_oracle as o
import workloads as wk


def test_noalloc_rejects_tensors_beyond_its_scratch_without_a_gpu():
    from epilogues_nvfp4_quantize_b200.build import build
    build()
    lib = ep.load()
    t = _lib._Tensor(16, 16, 16, 16385, 16384)
    # 16385 x 16384 values need one partial maximum more than the array holds
    assert lib.nvfp4_quantize_noalloc(16, 16385, 16384, 16384, 0, t, None) == 2
    t2 = _lib._Tensor(16, 16, 16, 128, 96)
    assert lib.nvfp4_quantize_noalloc(16, 128, 96, 96, 0, t2, None) == 2      # cols % 64
    assert lib.nvfp4_quantize_noalloc(None, 128, 64, 64, 0, t2, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("rows,cols,interleave", [(256, 1024, False), (130, 192, False), (768, 512, True)])
def test_noalloc_matches_workspace_quantiser_on_consecutive_calls(rows, cols, interleave):
    dev = torch.device("cuda", 0)
    for seed in (1, 2):  # two calls in a row share the static scratch
        x = wk.activations(rows, cols, 3, seed=seed + rows).to(dev)
        if seed == 2:
            x = x * 0.01  # a much smaller amax than the previous call left in the scratch
        ref = ep.NVFP4Tensor.empty(rows, cols, dev)
        ep.nvfp4_quantize(x, ref, compute_amax=True, interleave=interleave)
        got = ep.NVFP4Tensor.empty(rows, cols, dev)
        ep.nvfp4_quantize_noalloc(x, got, interleave=interleave)
        torch.cuda.synchronize()
        assert torch.equal(got.gscale, ref.gscale)
        assert torch.equal(got.codes, ref.codes)
        assert torch.equal(got.sf, ref.sf)
        # and against the oracle: the plain definition up to ties, the float32 order exactly
        from gpu_util import assert_nvfp4_plain, read_nvfp4
        xf = x.float().cpu().numpy()
        if interleave:
            xf = o.interleave_gate_up(xf)
        q, s, G, _ = read_nvfp4(got)
        assert G == o.global_scale(xf)
        assert_nvfp4_plain(q, s, xf, G, "noalloc")
        q32, s32, _ = o.quantize_fp32_order(xf)
        assert np.array_equal(q, q32) and np.array_equal(s, s32)
    assert ep.read_device_status() == 0
