"""Tensor-parallel sharding of the layer (host logic), on CPU: the index helpers are
partitions, and two gloo ranks computing their shards with the oracle reproduce the
unsharded layer (QKV and FFN-up column-parallel with no collective, FFN-down row-parallel
with one reduction)."""
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


@pytest.mark.parametrize("world", [1, 2, 4])
def test_shards_partition_rows_and_columns(world):
    n = 3 * HEADS * HD
    rows = np.concatenate([tp.qkv_shard_rows(HEADS, HD, world, r) for r in range(world)])
    assert np.array_equal(np.sort(rows), np.arange(n))
    # each rank's QKV shard: whole heads, Q then K then V
    r0 = tp.qkv_shard_rows(HEADS, HD, world, 0)
    assert np.all(r0.reshape(3, -1)[:, 0] % HD == 0)
    assert tp.qkv_shard_norm_cols(HEADS, HD, world) == 2 * len(r0) // 3
    up = np.concatenate([tp.ffn_up_shard_rows(NH, world, r) for r in range(world)])
    assert np.array_equal(np.sort(up), np.arange(2 * NH))
    u1 = tp.ffn_up_shard_rows(NH, world, world - 1)
    assert np.array_equal(u1[len(u1) // 2:], u1[:len(u1) // 2] + NH)  # gate j pairs with up j
    dn = np.concatenate([tp.ffn_down_shard_cols(NH, world, r) for r in range(world)])
    assert np.array_equal(dn, np.arange(NH))
    assert [tp.output_rows(M, world, r) for r in range(world)][-1].stop == M


def test_indivisible_splits_are_rejected():
    with pytest.raises(ValueError):
        tp.qkv_shard_rows(3, HD, 2, 0)
    with pytest.raises(ValueError):
        tp.ffn_down_shard_cols(NH, 3, 0)


def _inputs():
    a = wk.activations(M, K, 2, seed=1)
    wq = wk.weights(3 * HEADS * HD, K, 1 / np.sqrt(K), seed=2)
    wu = wk.weights(2 * NH, K, 1 / np.sqrt(K), seed=3)
    wd = wk.weights(K, NH, 1 / np.sqrt(NH), seed=4)
    wn_q, wn_k = wk.norm_weight(HD, 1, 3), wk.norm_weight(HD, 1, 5)
    return a, wq, wu, wd, wn_q, wn_k


def _layer(a, wq, wu, wd, wn_q, wn_k, rows_qkv=None, rows_up=None, cols_dn=None, world=1, G_h=None):
    """The layer's projections with the oracle, on a shard (or the whole layer). Shards
    keep the whole weights' per-tensor scales."""
    qq, sq, gq = o.quantized_operand(wq)
    qu, su, gu = o.quantized_operand(wu)
    qd, sd, gd = o.quantized_operand(wd)
    if rows_qkv is not None:
        qq, sq = qq[rows_qkv], sq[rows_qkv]
        qu, su = qu[rows_up], su[rows_up]
        qd, sd = qd[:, cols_dn], sd[:, cols_dn[::16] // 16]
    hr = HEADS // world
    w = np.concatenate([np.tile(wn_q, hr), np.tile(wn_k, hr)])
    c_qkv = o.gemm(o.dequantize(*o.quantize(o._as_f32(a), o.global_scale(o._as_f32(a)))),
                   o.dequantize(qq, sq, gq))
    qkv = o.rmsnorm_heads(c_qkv, w, HD, 2 * hr * HD, 1e-6)
    a_dec = o.dequantize(*o.quantize(o._as_f32(a), o.global_scale(o._as_f32(a))))
    h = o.bf16_round(o.swiglu(o.gemm(a_dec, o.dequantize(qu, su, gu))))
    if G_h is None:
        G_h = np.float32(np.abs(h).max() / 2688)
    qh, sh, _ = o.requantize(h, G_h)
    part = o.gemm(o.dequantize(qh, sh, G_h), o.dequantize(qd, sd, gd))
    return qkv, part, G_h


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, wq, wu, wd, wn_q, wn_k = _inputs()
        _, _, G_h = _layer(a, wq, wu, wd, wn_q, wn_k)  # the static scale of the whole h
        qkv, part, _ = _layer(a, wq, wu, wd, wn_q, wn_k,
                              tp.qkv_shard_rows(HEADS, HD, world, rank), tp.ffn_up_shard_rows(NH, world, rank),
                              tp.ffn_down_shard_cols(NH, world, rank), world, G_h)
        t = torch.from_numpy(part)
        dist.all_reduce(t)  # gloo has no reduce-scatter: reduce, then keep this rank's rows
        out = t.numpy()[tp.output_rows(M, world, rank)]
        np.save(os.path.join(out_dir, f"qkv{rank}.npy"), qkv)
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_reproduce_the_unsharded_layer(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    a, wq, wu, wd, wn_q, wn_k = _inputs()
    qkv_full, out_full, _ = _layer(a, wq, wu, wd, wn_q, wn_k)
    for r in range(world):
        rows = tp.qkv_shard_rows(HEADS, HD, world, r)
        # column-parallel: the rank's columns are exactly the unsharded layer's columns
        assert np.allclose(np.load(tmp_path / f"qkv{r}.npy"), qkv_full[:, rows], rtol=1e-12, atol=0)
        # row-parallel: the reduced partial sums are the unsharded output rows
        assert np.allclose(np.load(tmp_path / f"out{r}.npy"), out_full[tp.output_rows(M, world, r)],
                           rtol=1e-10, atol=1e-12)
