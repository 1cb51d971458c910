"""GPU parity of the row-parallel GEMM with its reduce-scatter in the epilogue
(gemm_nvfp4_reduce_rows_f32). Every destination lives on this GPU here: the kernel addresses a
peer-mapped destination exactly as a local one, and the world sizes, row splits and pitches
below cover its owner arithmetic. The reference is the pointwise GEMM's float32 output: the
reduce epilogue computes the same G_A G_B acc, and adding it into zero is exact. Both are
also checked against the oracle's float64 GEMM of the same codes: bit for bit on exactly
representable operands, within the tolerance otherwise."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_close, device, nvfp4_from_arrays, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed, exact):
    if exact:
        qa = wk.fp4_codes_exact(M, K, seed, 31)
        qb = wk.fp4_codes_exact(N, K, seed, 32)
        sa = o.e4m3_encode(wk.pow2_scales_exact(M, K // 16, seed, 33).astype(np.float32))
        sb = o.e4m3_encode(wk.pow2_scales_exact(N, K // 16, seed, 34).astype(np.float32))
        return nvfp4_from_arrays(qa, sa, 0.5), nvfp4_from_arrays(qb, sb, 0.25)
    a = wk.activations(M, K, wk.outlier_count(K), seed=seed)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=seed)
    return quantize_gpu(a), quantize_gpu(b)


# (world, rows per rank, N, K, exact operands): M % 256 == 0, M % 256 == 128 (the last pair
# tile half past M) and M = 128 (the single-CTA kernel); 128 rows per rank puts the two
# halves of a pair tile on two ranks
@pytest.mark.parametrize("world,rpr,N,K,exact", [(1, 256, 512, 512, True), (2, 256, 512, 1024, True),
                                                 (4, 128, 768, 512, True), (1, 384, 256, 256, True),
                                                 (3, 384, 512, 512, True), (2, 1024, 1536, 1024, False),
                                                 (1, 128, 512, 512, True)])
def test_reduce_rows_equals_pointwise_f32(world, rpr, N, K, exact):
    M = world * rpr
    A, B = _operands(M, N, K, seed=world * 100 + rpr, exact=exact)
    ref = torch.empty(M, N, dtype=torch.float32, device=device())
    ep.gemm_nvfp4_pointwise(A, B, ref)
    ldd = N + 4 * (world % 2)  # a padded pitch for odd world sizes
    outs = [torch.zeros(rpr, ldd, dtype=torch.float32, device=device()) for _ in range(world)]
    ptrs = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device=device())
    ep.gemm_nvfp4_reduce_rows_f32(A, B, ptrs, rpr, ldd)
    torch.cuda.synchronize()
    for r in range(world):
        assert torch.equal(outs[r][:, :N], ref[r * rpr:(r + 1) * rpr]), f"destination {r}"
        if ldd > N:
            assert torch.all(outs[r][:, N:] == 0), "columns past N are untouched"
    # the oracle's float64 GEMM of the same codes and scales
    qa, sa, ga, _ = read_nvfp4(A)
    qb, sb, gb, _ = read_nvfp4(B)
    full = o.gemm(o.dequantize(qa, sa, ga), o.dequantize(qb, sb, gb))
    got = np.concatenate([t[:, :N].cpu().numpy() for t in outs]).astype(np.float64)
    if exact:
        assert np.array_equal(got, full.astype(np.float32).astype(np.float64))
    else:
        assert_close(got, full, "reduce rows vs oracle")
    # a second call adds the same values again: exactly twice the first result
    ep.gemm_nvfp4_reduce_rows_f32(A, B, ptrs, rpr, ldd)
    torch.cuda.synchronize()
    for r in range(world):
        assert torch.equal(outs[r][:, :N], 2 * ref[r * rpr:(r + 1) * rpr]), f"destination {r}, second call"
    assert ep.read_device_status() == 0


def test_reduce_rows_sums_k_slices_into_the_full_product():
    """The use it exists for: two K slices of one product (two ranks' shards of a row-parallel
    GEMM), each reduced into the same destinations, add up to the unsharded product."""
    M, N, K, world = 512, 512, 1024, 2
    A, B = _operands(M, N, K, seed=5, exact=True)
    qa, sa, _, _ = _read(A)
    qb, sb, _, _ = _read(B)
    full = o.gemm(o.dequantize(qa, sa, 0.5), o.dequantize(qb, sb, 0.25))
    rpr = M // world
    outs = [torch.zeros(rpr, N, dtype=torch.float32, device=device()) for _ in range(world)]
    ptrs = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device=device())
    for k0 in (0, K // 2):
        As = nvfp4_from_arrays(qa[:, k0:k0 + K // 2], sa[:, k0 // 16:(k0 + K // 2) // 16], 0.5)
        Bs = nvfp4_from_arrays(qb[:, k0:k0 + K // 2], sb[:, k0 // 16:(k0 + K // 2) // 16], 0.25)
        ep.gemm_nvfp4_reduce_rows_f32(As, Bs, ptrs, rpr, N)
    torch.cuda.synchronize()
    got = np.concatenate([t.cpu().numpy() for t in outs]).astype(np.float64)
    assert np.array_equal(got, full), "the two K slices must add up to the exact product"


def _read(t):
    from gpu_util import read_nvfp4
    return read_nvfp4(t)


def test_reduce_rows_misaligned_destination_is_reported_not_dereferenced():
    """A destination pointer that is not 16-byte aligned cannot be checked on the host (the
    pointer array is device memory): the kernel reports it in the device status word and
    leaves that block alone; the aligned destination is still written."""
    M, N, K = 256, 256, 256
    A, B = _operands(M, N, K, seed=9, exact=True)
    ref = torch.empty(M, N, dtype=torch.float32, device=device())
    ep.gemm_nvfp4_pointwise(A, B, ref)
    good = torch.zeros(128, N, dtype=torch.float32, device=device())
    backing = torch.zeros(128 * N + 4, dtype=torch.float32, device=device())
    bad_ptr = backing.data_ptr() + 4  # 4-byte offset: misaligned for the 16-byte additions
    ptrs = torch.tensor([good.data_ptr(), bad_ptr], dtype=torch.int64, device=device())
    ep.gemm_nvfp4_reduce_rows_f32(A, B, ptrs, 128, N)
    assert ep.read_device_status() == 3  # NVFP4_ERR_MISALIGNED
    assert torch.equal(good, ref[:128])
    assert torch.all(backing == 0)
    assert ep.read_device_status() == 0  # reading clears it
