"""GPU parity of gemm_nvfp4_pointwise (bias, ReLU, cast to bf16/f16/f32, optional NVFP4
output for the next layer) against the oracle. Exactly representable operands make the
FP32 accumulator exact, so the outputs are compared bit for bit; general operands within
the benchmark spec's tolerance. From M = 256 on the CTA-pair kernel runs (for M % 256 == 128 with
its last tile half past M); M = 128 runs the single-CTA kernel."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_close, assert_nvfp4_plain, device, nvfp4_from_arrays, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


def _exact_operands(M, N, K, seed):
    qa = wk.fp4_codes_exact(M, K, seed, 31)
    qb = wk.fp4_codes_exact(N, K, seed, 32)
    sa = o.e4m3_encode(wk.pow2_scales_exact(M, K // 16, seed, 33).astype(np.float32))
    sb = o.e4m3_encode(wk.pow2_scales_exact(N, K // 16, seed, 34).astype(np.float32))
    return qa, sa, qb, sb


def _cast(y, dtype):
    if dtype == torch.float32:
        return y.astype(np.float32)
    if dtype == torch.float16:
        return y.astype(np.float16)
    return o.bf16_round(y).astype(np.float32)


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (384, 768, 1024), (2048, 2560, 256)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("relu", [False, True])
def test_pointwise_is_exact_on_exactly_representable_inputs(M, N, K, dtype, relu):
    qa, sa, qb, sb = _exact_operands(M, N, K, seed=M + K)
    A, B = nvfp4_from_arrays(qa, sa, 1.0), nvfp4_from_arrays(qb, sb, 0.5)
    # a full-mantissa bias: alpha*acc + bias is rounded once, to float32
    bias = (np.random.default_rng(N).standard_normal(N) * 2.0).astype(np.float32)
    D = torch.empty(M, N, dtype=dtype, device=device())
    ep.gemm_nvfp4_pointwise(A, B, D, bias=torch.from_numpy(bias).to(device()), relu=relu)
    c = 0.5 * o.gemm(o.dequantize(qa, sa, 1.0), o.dequantize(qb, sb, 1.0))
    want = _cast(o.pointwise(c, bias, relu), dtype)
    got = D.float().cpu().numpy() if dtype != torch.float32 else D.cpu().numpy()
    assert np.array_equal(got.astype(np.float32), want.astype(np.float32)), \
        f"{int((got != want).sum())} of {got.size} outputs differ"


@pytest.mark.parametrize("M", [256, 384])
def test_pointwise_matches_oracle_on_workload_inputs(M):
    K, N = 1024, 768
    a = wk.activations(M, K, 2, seed=M)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=M)
    bias = (0.1 * np.random.default_rng(M).standard_normal(N)).astype(np.float32)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_pointwise(quantize_gpu(a), quantize_gpu(b), D, bias=torch.from_numpy(bias).to(device()), relu=True)
    ref = o.bf16_round(o.problem_pointwise(a, b, bias, relu=True))
    assert_close(D.float().cpu().numpy(), ref, "pointwise bias+relu bf16")


@pytest.mark.parametrize("M", [256, 128])
def test_pointwise_nvfp4_output_equals_quantize_of_bf16_output(M):
    """The fused next-layer quantisation is nvfp4_quantize (static scale) of the bf16
    output, bit for bit; also without D."""
    K, N = 512, 1024
    a = wk.activations(M, K, 1, seed=7)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=8)
    A, B = quantize_gpu(a), quantize_gpu(b)
    bias = torch.from_numpy((0.05 * np.random.default_rng(3).standard_normal(N)).astype(np.float32)).to(device())
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_pointwise(A, B, D, bias=bias)
    G = float(D.float().abs().max().item()) / 2688
    Dq = ep.NVFP4Tensor.empty(M, N, device())
    Dq.gscale.fill_(G)
    ep.gemm_nvfp4_pointwise(A, B, D, bias=bias, Dq=Dq)
    t = ep.NVFP4Tensor.empty(M, N, device())
    t.gscale.fill_(G)
    ep.nvfp4_quantize(D, t, compute_amax=False)
    q1, s1, _, b1 = read_nvfp4(Dq)
    q2, s2, _, b2 = read_nvfp4(t)
    assert np.array_equal(q1, q2) and np.array_equal(b1, b2)
    # and against the oracle: the plain quantisation of the bf16 output, up to ties
    assert_nvfp4_plain(q1, s1, D.float().cpu().numpy(), np.float32(G), "pointwise nvfp4 output")
    Dq2 = ep.NVFP4Tensor.empty(M, N, device())
    Dq2.gscale.fill_(G)
    ep.gemm_nvfp4_pointwise(A, B, None, bias=bias, Dq=Dq2)
    q3, _, _, b3 = read_nvfp4(Dq2)
    assert np.array_equal(q3, q1) and np.array_equal(b3, b1)


def test_pointwise_argument_errors():
    qa, sa, qb, sb = _exact_operands(128, 256, 256, seed=1)
    A, B = nvfp4_from_arrays(qa, sa, 1.0), nvfp4_from_arrays(qb, sb, 1.0)
    with pytest.raises(RuntimeError):
        ep.gemm_nvfp4_pointwise(A, B, None)  # neither D nor Dq
    D = torch.empty(128, 256, dtype=torch.float32, device=device())
    misaligned = torch.zeros(257, dtype=torch.float32, device=device())[1:]
    with pytest.raises(RuntimeError):
        ep.gemm_nvfp4_pointwise(A, B, D, bias=misaligned)
    assert ep.read_device_status() == 0
