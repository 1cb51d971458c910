"""Tensor-parallel sharding of a DiT layer's projections over the ranks of a
torch.distributed group.

Every output tile of the fused GEMMs is independent ("Serving sub-second Ideogram v4
without quality loss", section "Epilogue fusion in brief"), so the layer shards without
touching the epilogues:

- QKV, column-parallel on head boundaries: rank r owns heads [r h/w, (r+1) h/w) of each
  of the Q, K and V blocks. Its weight rows are those heads of Q, then of K, then of V, so
  the fused RMSNorm sees Q and K heads first (n_norm_cols = 2 N_q / w) and V passes through.
  No collective.
- FFN-up, column-parallel on gate/up pairs: rank r owns intermediate columns
  [r Nh/w, (r+1) Nh/w) of both the gate and the up half; its shard is interleaved as a
  whole, so SwiGLU stays inside each thread. No collective.
- FFN-down, row-parallel: rank r multiplies its intermediate columns by the matching K
  slice of the down weight; the partial sums over the ranks are added up, leaving rank r
  the output rows [r M/w, (r+1) M/w). Two ways:
  - reduce="nccl": the GEMM writes its partials (pointwise epilogue: float32 by default, or
    bf16 with partials="bf16", half the NVLink bytes at one bf16 rounding per rank), then
    one NCCL reduce-scatter over the token rows;
  - reduce="fused": the GEMM's epilogue adds each partial row straight into its owner's
    output block (gemm_nvfp4_reduce_rows_f32). The blocks are symmetric memory, so every
    rank holds the others' addresses. A barrier before the GEMM means every block is
    zeroed; a barrier after it means every addition has landed. The barrier is the
    library's own kernel (nvfp4_signal_barrier) on peer-mapped signal words: its waits are
    bounded, and a rank that never arrives ends the others' wait with a status in the
    device status word, leaving their GPUs usable. The only traffic between GPUs is those
    stores and signal words: no kernel loads data from another GPU's memory.

The index helpers below are pure host logic (tested with gloo ranks on the CPU); TPLayer
runs them with the library's kernels and NCCL or symmetric memory.
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def _check_split(n: int, world: int, what: str) -> int:
    if world < 1 or n % world:
        raise ValueError(f"{what} = {n} does not split over {world} ranks")
    return n // world


def qkv_shard_rows(heads: int, head_dim: int, world: int, rank: int) -> np.ndarray:
    """Rows of the [Q | K | V] weight (3 * heads * head_dim rows) owned by `rank`: its
    heads of Q, then of K, then of V."""
    hr = _check_split(heads, world, "heads")
    blk = heads * head_dim
    own = np.arange(rank * hr * head_dim, (rank + 1) * hr * head_dim)
    return np.concatenate([own, blk + own, 2 * blk + own])


def qkv_shard_norm_cols(heads: int, head_dim: int, world: int) -> int:
    """Normalised (Q and K) columns of a rank's QKV shard."""
    return 2 * _check_split(heads, world, "heads") * head_dim


def ffn_up_shard_rows(nh: int, world: int, rank: int) -> np.ndarray:
    """Rows of the logical [gate | up] weight (2 * nh rows) owned by `rank`: its gate rows,
    then the matching up rows, i.e. a [gate | up] weight of its own."""
    c = _check_split(nh, world, "intermediate size")
    own = np.arange(rank * c, (rank + 1) * c)
    return np.concatenate([own, nh + own])


def ffn_down_shard_cols(nh: int, world: int, rank: int) -> np.ndarray:
    """K columns of the down weight (and columns of the intermediate activation) owned by
    `rank`."""
    c = _check_split(nh, world, "intermediate size")
    return np.arange(rank * c, (rank + 1) * c)


def output_rows(m: int, world: int, rank: int) -> slice:
    """Rows of the down-projection output a rank holds after the reduce-scatter."""
    r = _check_split(m, world, "token rows")
    return slice(rank * r, (rank + 1) * r)


class TPLayer:
    """One DiT layer's projections sharded over a process group (one rank per GPU).

    Weights are given whole (bf16, on this rank's device) and sharded here; each rank
    packs only its shard. step(xq) takes the NVFP4 activations (replicated, M x K) and
    returns (qkv_local bf16 M x 3*(heads/w)*head_dim, out_rows (M/w) x K: float32, or bf16
    with reduce="nccl", partials="bf16").
    With reduce="fused", out_rows is this rank's symmetric-memory block for that M: the next
    step of the same M zeroes and refills it, so copy it out to keep it."""

    def __init__(self, w_qkv, w_up, w_down, w_norm_q, w_norm_k, heads: int, head_dim: int,
                 h_gscale: float, group=None, eps: float = 1e-6, reduce: str = "nccl",
                 partials: str = "f32"):
        import torch
        import torch.distributed as dist
        from . import _lib as L

        self.dist, self.torch, self.L = dist, torch, L
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        dev = w_qkv.device
        self.heads, self.head_dim, self.eps = heads, head_dim, eps
        nh = w_up.shape[0] // 2
        rows_qkv = torch.from_numpy(qkv_shard_rows(heads, head_dim, self.world, self.rank)).to(dev)
        rows_up = torch.from_numpy(ffn_up_shard_rows(nh, self.world, self.rank)).to(dev)
        cols_dn = torch.from_numpy(ffn_down_shard_cols(nh, self.world, self.rank)).to(dev)
        self.n_norm = qkv_shard_norm_cols(heads, head_dim, self.world)
        # Each shard is quantised with the per-tensor scale of the whole weight, so that its
        # codes and block scales (blocks of 16 along K) are exactly those of the unsharded
        # weight: the sharded layer computes what the unsharded one does.
        self.Wqkv = self._pack(w_qkv, w_qkv.index_select(0, rows_qkv).contiguous())
        self.Wup = self._pack(w_up, w_up.index_select(0, rows_up).contiguous(), interleave=True)
        self.Wdown = self._pack(w_down, w_down.index_select(1, cols_dn).contiguous())
        hr = heads // self.world
        self.w_norm = torch.cat([w_norm_q.repeat(hr), w_norm_k.repeat(hr)]).float().contiguous().to(dev)
        self.h_gscale = float(h_gscale)
        self.nh_local = nh // self.world
        if reduce not in ("nccl", "fused"):
            raise ValueError(f"reduce must be 'nccl' or 'fused', not {reduce!r}")
        self.reduce = reduce
        if partials not in ("f32", "bf16"):
            raise ValueError(f"partials must be 'f32' or 'bf16', not {partials!r}")
        self.partial_dtype = torch.float32 if partials == "f32" else torch.bfloat16
        self._fused = {}  # M -> (this rank's output block, signal-array pointers or None, block pointers)
        self._epoch = 0   # barriers taken so far (the signal words count them)
        self.barrier_limit_ns = 10_000_000_000

    def _pack(self, whole, shard, interleave: bool = False):
        T, L = self.L.NVFP4Tensor, self.L
        dev = whole.device
        full = L.nvfp4_quantize(whole, T.empty(whole.shape[0], whole.shape[1], dev))  # for its G only
        out = T.empty(shard.shape[0], shard.shape[1], dev)
        out.gscale.copy_(full.gscale)
        return L.nvfp4_quantize(shard, out, compute_amax=False, interleave=interleave)

    def step(self, xq, qkv: Optional["object"] = None):
        torch, L = self.torch, self.L
        M = xq.rows
        dev = xq.codes.device
        if qkv is None:
            qkv = torch.empty(M, self.Wqkv.rows, dtype=torch.bfloat16, device=dev)
        L.gemm_nvfp4_rmsnorm(xq, self.Wqkv, self.w_norm, self.head_dim, self.n_norm, self.eps, qkv)
        h = L.NVFP4Tensor.empty(M, self.nh_local, dev)
        h.gscale.fill_(self.h_gscale)  # static scale, the same on every rank
        L.gemm_nvfp4_swiglu(xq, self.Wup, None, h)
        if self.reduce == "fused":
            out, sig, ptrs = self._fused_block(M, dev)
            out.zero_()
            self._barrier(sig)  # every rank's block is zeroed before any rank adds into it
            L.gemm_nvfp4_reduce_rows_f32(h, self.Wdown, ptrs, M // self.world, self.Wdown.rows)
            self._barrier(sig)  # every rank's additions have landed
            return qkv, out
        part = torch.empty(M, self.Wdown.rows, dtype=self.partial_dtype, device=dev)
        L.gemm_nvfp4_pointwise(h, self.Wdown, part)
        out = torch.empty(M // self.world, self.Wdown.rows, dtype=self.partial_dtype, device=dev)
        if self.world > 1:
            self.dist.reduce_scatter_tensor(out, part, group=self.group)
        else:
            out = part
        return qkv, out

    def _fused_block(self, M: int, dev):
        """This rank's (M/w) x N float32 output block and every rank's block address, made
        once per M. With more than one rank the blocks are symmetric memory: each rank maps
        the others' blocks and receives their addresses at the rendezvous."""
        if M not in self._fused:
            torch = self.torch
            rows = output_rows(M, self.world, self.rank)
            n = self.Wdown.rows
            if self.world > 1:
                import torch.distributed._symmetric_memory as symm_mem
                group = self.group if self.group is not None else self.dist.group.WORLD
                block = symm_mem.empty((rows.stop - rows.start, n), dtype=torch.float32, device=dev)
                hdl = symm_mem.rendezvous(block, group)
                ptrs = torch.tensor(list(hdl.buffer_ptrs), dtype=torch.int64, device=dev)
                # one uint32 signal word per rank, in symmetric memory too, zeroed on every
                # rank before any rank's first barrier
                words = symm_mem.empty((self.world,), dtype=torch.int32, device=dev)
                words.zero_()
                shdl = symm_mem.rendezvous(words, group)
                sig = (words, torch.tensor(list(shdl.buffer_ptrs), dtype=torch.int64, device=dev))
                torch.cuda.synchronize(dev)
                self.dist.barrier(group=self.group)
            else:
                block = torch.empty(rows.stop - rows.start, n, dtype=torch.float32, device=dev)
                sig = None
                ptrs = torch.tensor([block.data_ptr()], dtype=torch.int64, device=dev)
            self._fused[M] = (block, sig, ptrs)
        return self._fused[M]

    def _barrier(self, sig):
        """Stream-ordered barrier over the ranks' signal words (nothing to wait for at world
        size 1): the library's bounded barrier kernel. A rank that never arrives ends the
        others' wait after barrier_limit_ns with NVFP4_ERR_DEVICE_TIMEOUT in their device
        status words; their kernels return and their contexts stay usable."""
        if sig is not None:
            self._epoch += 1
            self.L.signal_barrier(sig[1], self.rank, self._epoch, self.barrier_limit_ns)
