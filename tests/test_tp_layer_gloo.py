"""TPLayer itself on two gloo ranks (CPU): the sharding, the packing with the whole weights'
per-tensor scales, the static scale of h, the partial sums and the reduce-scatter, run end
to end. The library's kernels are replaced by a test double that computes each call with
the oracle on CPU tensors (the kernels' own parity is covered by the GPU tests); the ranks'
results must equal one unsharded TPLayer's: QKV columns bit for bit, output rows up to the
rounding of adding two partial sums (float32, or bf16 partials)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from epilogues_nvfp4_quantize_b200 import parallel as tp
from oracle import nvfp4_oracle as o
import workloads as wk

HEADS, HD, K, NH, M = 4, 128, 256, 512, 64


class FakeNVFP4:
    """An NVFP4 tensor of the test double: codes and scales as arrays, G as a tensor."""

    def __init__(self, rows, cols, device="cpu"):
        self.rows, self.cols = rows, cols
        self.codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        self.gscale = torch.zeros((1,), dtype=torch.float32, device=device)
        self.q = self.s = None

    @classmethod
    def empty(cls, rows, cols, device="cpu"):
        return cls(rows, cols, device)

    def values(self):
        return o.dequantize(self.q, self.s, np.float32(self.gscale.item()))


class FakeLib:
    """The calls TPLayer makes, computed with the oracle (float32 evaluation order, as the
    kernels take their rounding decisions)."""
    NVFP4Tensor = FakeNVFP4

    @staticmethod
    def nvfp4_quantize(x, out, compute_amax=True, interleave=False, workspace=None, stream=None):
        xf = x.float().numpy()
        if interleave:
            xf = o.interleave_gate_up(xf)
        G = None if compute_amax else np.float32(out.gscale.item())
        out.q, out.s, g = o.quantize_fp32_order(xf, G)
        out.gscale.fill_(float(g))
        return out

    @staticmethod
    def gemm_nvfp4_rmsnorm(A, B, w, head_dim, n_norm_cols, eps, D, stream=None):
        c = o.gemm(A.values(), B.values())
        D.copy_(torch.from_numpy(o.rmsnorm_heads(c, w.numpy().astype(np.float64), head_dim, n_norm_cols, eps)))
        return D

    @staticmethod
    def gemm_nvfp4_swiglu(A, B, D=None, Dq=None, stream=None):
        c = o.gemm(A.values(), B.values())  # columns interleaved: gate j, up j
        h = o.bf16_round(o.swiglu(np.concatenate([c[:, 0::2], c[:, 1::2]], axis=1)))
        if D is not None:
            D.copy_(torch.from_numpy(h))
        if Dq is not None:
            Dq.q, Dq.s, _ = o.requantize(h, np.float32(Dq.gscale.item()))
        return D, Dq

    @staticmethod
    def gemm_nvfp4_pointwise(A, B, D=None, bias=None, relu=False, Dq=None, stream=None):
        D.copy_(torch.from_numpy(o.gemm(A.values(), B.values())))
        return D, Dq


def _weights():
    wq = wk.weights(3 * HEADS * HD, K, 1 / np.sqrt(K), seed=2)
    wu = wk.weights(2 * NH, K, 1 / np.sqrt(K), seed=3)
    wd = wk.weights(K, NH, 1 / np.sqrt(NH), seed=4)
    wn_q = torch.from_numpy(wk.norm_weight(HD, 1, 3).astype(np.float32))
    wn_k = torch.from_numpy(wk.norm_weight(HD, 1, 5).astype(np.float32))
    return wq, wu, wd, wn_q, wn_k


def _run_layer(h_gscale, partials="f32"):
    """One step of TPLayer (this process's world) on the fixed inputs, with the double."""
    from epilogues_nvfp4_quantize_b200 import _lib
    for name in ("NVFP4Tensor", "nvfp4_quantize", "gemm_nvfp4_rmsnorm", "gemm_nvfp4_swiglu",
                 "gemm_nvfp4_pointwise"):
        setattr(_lib, name, getattr(FakeLib, name))
    wq, wu, wd, wn_q, wn_k = _weights()
    layer = tp.TPLayer(wq, wu, wd, wn_q, wn_k, HEADS, HD, h_gscale, reduce="nccl", partials=partials)
    xq = FakeLib.nvfp4_quantize(wk.activations(M, K, 2, seed=1), FakeNVFP4(M, K))
    qkv, out = layer.step(xq)
    return qkv.float().numpy(), out.float().numpy()


def _h_gscale():
    """The static scale of the whole h, from the unsharded layer (as a calibration would)."""
    wq, wu, wd, wn_q, wn_k = _weights()
    a = FakeLib.nvfp4_quantize(wk.activations(M, K, 2, seed=1), FakeNVFP4(M, K))
    b = FakeLib.nvfp4_quantize(wu, FakeNVFP4(2 * NH, K))
    c = o.gemm(a.values(), b.values())
    h = o.bf16_round(o.swiglu(c))
    return float(np.abs(h).max() / 2688)


def _rank_main(rank, world, port, out_dir, partials):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        qkv, out = _run_layer(_h_gscale(), partials)
        np.save(os.path.join(out_dir, f"qkv{rank}.npy"), qkv)
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _unsharded(partials):
    """world 1 in a child process (the double replaces library functions for the process)."""
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(1, _free_port(), d, partials), nprocs=1, start_method="spawn")
        return np.load(os.path.join(d, "qkv0.npy")), np.load(os.path.join(d, "out0.npy"))


@pytest.mark.parametrize("partials", ["f32", "bf16"])
def test_tplayer_on_two_gloo_ranks_equals_the_unsharded_layer(tmp_path, partials):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), partials), nprocs=world,
                       start_method="spawn")
    qkv_full, out_full = _unsharded(partials)
    assert qkv_full.shape == (M, 3 * HEADS * HD) and out_full.shape == (M, K)
    for r in range(world):
        # column-parallel QKV: the rank's columns are the unsharded layer's, bit for bit
        cols = tp.qkv_shard_rows(HEADS, HD, world, r)
        assert np.array_equal(np.load(tmp_path / f"qkv{r}.npy"), qkv_full[:, cols])
        # row-parallel FFN-down: the reduce-scatter leaves rank r the output rows it owns
        got = np.load(tmp_path / f"out{r}.npy")
        ref = out_full[tp.output_rows(M, world, r)]
        assert got.shape == (M // world, K)
        rms = np.sqrt(np.mean(ref * ref))
        if partials == "f32":
            # two float32 partials added in float32
            assert np.all(np.abs(got - ref) <= 2e-6 * (np.abs(ref) + rms))
        else:
            # each partial rounded to bf16 and their bf16 sum rounded again, against one
            # rounding of the whole sum; a rounding to bf16 (8 significant bits) moves a
            # value by at most 2^-8 of itself: 2^-8 (|got| + |ref|) for the two sums, and
            # 2^-8 (|p0| + |p1|) for the partials, which stay under 4 rms together here
            assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 2.0 ** -6 * rms)
