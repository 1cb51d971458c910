"""GPU parity of the fused GEMM entry points against the oracle, at sizes the oracle
finishes in seconds that still span several tiles, several tiles per CTA, and the
degenerate cases (one tile, one K step, no normalised columns). From M = 256 on the CTA-pair
kernel runs; for M % 256 == 128 its last tile's second CTA lies past M (rows 384, 1152, ...
below). M = 128 runs the single-CTA kernel. Each appears with more tiles than the GPU has SMs
(pairs) in at least one case."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import (assert_close, assert_requant_point13, bf16_bits, bf16_to_np, device, level_index,
                      nvfp4_from_arrays, quantize_gpu, read_nvfp4, rel_err, REL_TOL)

pytestmark = pytest.mark.gpu


def _exact_operands(M, N, K, seed):
    qa = wk.fp4_codes_exact(M, K, seed, 21)
    qb = wk.fp4_codes_exact(N, K, seed, 22)
    sa = o.e4m3_encode(wk.pow2_scales_exact(M, K // 16, seed, 23).astype(np.float32))
    sb = o.e4m3_encode(wk.pow2_scales_exact(N, K // 16, seed, 24).astype(np.float32))
    return qa, sa, qb, sb


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (384, 768, 3072), (2048, 2560, 256),
                                   (1152, 4352, 256), (512, 256, 3072)])
def test_plain_gemm_is_exact_on_exactly_representable_inputs(M, N, K):
    """E2M1 codes x power-of-two scales: every partial sum is a multiple of 2^-6 below
    2^24 * 2^-6, so FP32 accumulation is exact in any order and the bf16 output must be
    the round-to-nearest-even of the exact product, bit for bit. This pins the operand
    layout, the scale-factor layout and the MMA kind."""
    qa, sa, qb, sb = _exact_operands(M, N, K, seed=M + N + K)
    A = nvfp4_from_arrays(qa, sa, 1.0)
    B = nvfp4_from_arrays(qb, sb, 1.0)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_plain(A, B, D)
    ref = o.bf16_round(o.gemm(o.dequantize(qa, sa, 1.0), o.dequantize(qb, sb, 1.0)))
    got = bf16_bits(D)
    want = o.bf16_bits(ref)
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} outputs differ"


@pytest.mark.parametrize("M,N,K", [(8192, 5120, 1024), (8064, 5120, 1024), (128, 512, 4096)])
def test_plain_gemm_exact_over_many_ring_wraps(M, N, K):
    """Many K steps per CTA (or CTA pair) through the rings: about 35 in the 5-stage ring with
    4 TMEM scale slots of the CTA pair (M = 8192, 4 K steps per tile; M = 8064 adds a last
    tile half past M), and 16 in the 3-stage ring with 3 slots of the single CTA (M = 128,
    one tile per CTA). The stage and slot counters wrap against each other and across tile
    boundaries. Exactly representable inputs make every output bit-exact; rows are sampled,
    always including the first and the last."""
    qa, sa, qb, sb = _exact_operands(M, N, K, seed=77)
    A = nvfp4_from_arrays(qa, sa, 1.0)
    B = nvfp4_from_arrays(qb, sb, 1.0)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_plain(A, B, D)
    rng = np.random.default_rng(M)
    n = min(256, M)
    rows = np.sort(np.concatenate([[0, M - 1], rng.choice(np.arange(1, M - 1), size=n - 2, replace=False)]))
    ref = o.bf16_round(o.gemm(o.dequantize(qa[rows], sa[rows], 1.0), o.dequantize(qb, sb, 1.0)))
    got = bf16_bits(D[torch.from_numpy(rows).to(device())])
    want = o.bf16_bits(ref)
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} outputs differ"
    assert ep.read_device_status() == 0


def test_plain_gemm_scales_by_both_global_scales():
    M, N, K = 128, 256, 512
    qa, sa, qb, sb = _exact_operands(M, N, K, seed=5)
    A = nvfp4_from_arrays(qa, sa, 0.5)
    B = nvfp4_from_arrays(qb, sb, 0.25)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_plain(A, B, D)
    ref = o.bf16_round(o.gemm(o.dequantize(qa, sa, 0.5), o.dequantize(qb, sb, 0.25)))
    assert np.array_equal(bf16_bits(D), o.bf16_bits(ref))


@pytest.mark.parametrize("M,N,K,ldd", [(256, 512, 512, 512), (1280, 768, 768, 800), (2048, 2560, 512, 2560),
                                       (384, 512, 512, 512), (1152, 4352, 256, 4352)])
def test_plain_gemm_matches_oracle(M, N, K, ldd):
    a = wk.activations(M, K, wk.outlier_count(K), seed=1)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=1)
    A, B = quantize_gpu(a), quantize_gpu(b)
    Dfull = torch.full((M, ldd), 7.0, dtype=torch.bfloat16, device=device())
    D = Dfull[:, :N]
    ep.gemm_nvfp4_plain(A, B, D)
    assert_close(bf16_to_np(D), o.problem_plain(a, b), "plain")
    if ldd > N:  # the columns past N of each row are untouched
        assert torch.all(Dfull[:, N:] == 7.0)


def _rmsnorm_case(M, K, N, hd, n_norm, seed=0, eps=1e-6):
    a = wk.activations(M, K, wk.outlier_count(K), seed=seed)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=seed)
    w = np.tile(wk.norm_weight(hd, seed), max(n_norm // hd, 1))[:n_norm].astype(np.float32)
    A, B = quantize_gpu(a), quantize_gpu(b)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    wt = torch.from_numpy(w).to(device()) if n_norm else None
    ep.gemm_nvfp4_rmsnorm(A, B, wt, hd, n_norm, eps, D)
    ref = o.problem_rmsnorm(a, b, w, hd, n_norm, eps)
    return bf16_to_np(D), ref


@pytest.mark.parametrize("M,K,N,hd,n_norm", [
    (256, 1024, 1024, 256, 1024),   # the tiny QK-norm case: 4 heads of 256, all normalised
    (256, 512, 768, 256, 512),      # V block passes through
    (256, 512, 768, 128, 384),      # 128-wide heads, normalised part ends mid-tile
    (384, 256, 512, 128, 0),        # nothing normalised
    (2048, 512, 2560, 256, 1536),   # several tiles per CTA
    (128, 512, 768, 256, 512),      # the single-CTA kernel
    (1152, 512, 1024, 256, 768),    # the pair kernel's last tile half past M
])
def test_rmsnorm_gemm_matches_oracle(M, K, N, hd, n_norm):
    got, ref = _rmsnorm_case(M, K, N, hd, n_norm)
    assert_close(got, ref, f"rmsnorm hd{hd}")


def test_rmsnorm_output_has_unit_rms_per_head_before_weight():
    M, K, N, hd = 256, 512, 512, 256
    a = wk.activations(M, K, 1, seed=3)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=3)
    A, B = quantize_gpu(a), quantize_gpu(b)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_rmsnorm(A, B, torch.ones(N, device=device()), hd, N, 0.0, D)
    y = bf16_to_np(D).reshape(M, N // hd, hd)
    rms = np.sqrt(np.mean(y * y, axis=2))
    np.testing.assert_allclose(rms, 1.0, rtol=4e-3)


def _swiglu_case(M, K, nh, seed=0, requant=True, write_d=True):
    a = wk.activations(M, K, wk.outlier_count(K), seed=seed)
    b = wk.weights(2 * nh, K, 1 / np.sqrt(K), seed=seed)     # logical [gate | up]
    A = quantize_gpu(a)
    B = quantize_gpu(b, interleave=True)
    ref = o.problem_swiglu(a, b)
    G = np.float32(np.abs(ref).max() / 2688)                 # static scale of the output
    D = torch.empty(M, nh, dtype=torch.bfloat16, device=device()) if write_d else None
    Dq = None
    if requant:
        Dq = ep.NVFP4Tensor.empty(M, nh, device())
        Dq.gscale.fill_(float(G))
    ep.gemm_nvfp4_swiglu(A, B, D, Dq)
    return a, b, ref, G, D, Dq


@pytest.mark.parametrize("M,K,nh", [(128, 256, 128), (256, 512, 512), (2048, 512, 1280), (640, 512, 384)])
def test_swiglu_gemm_matches_oracle(M, K, nh):
    a, b, ref, G, D, Dq = _swiglu_case(M, K, nh)
    got = bf16_to_np(D)
    assert_close(got, ref, "swiglu")
    # re-quantised output, code for code: the plain re-quantisation of the GPU's own bf16
    # output up to ties; against the oracle's re-quantisation of its own bf16 result, a
    # code or scale may differ only where the two bf16 values differ, by one level (one
    # scale code)
    q, s, Gq, _ = read_nvfp4(Dq)
    assert Gq == G
    assert assert_requant_point13(q, s, got, ref, G, "swiglu requant") < 0.01


@pytest.mark.parametrize("M", [512, 384])
def test_fused_requant_equals_quantize_of_fused_bf16(M):
    """GPU invariant: the re-quantised output is nvfp4_quantize (static scale) applied to
    the fused bf16 output, bit for bit (M = 384: the last pair tile half past M, whose
    re-quantised rows must not be written)."""
    a, b, ref, G, D, Dq = _swiglu_case(M, 768, 768, seed=4)
    t = ep.NVFP4Tensor.empty(M, 768, device())
    t.gscale.fill_(float(G))
    ep.nvfp4_quantize(D, t, compute_amax=False)
    q1, s1, _, b1 = read_nvfp4(Dq)
    q2, s2, _, b2 = read_nvfp4(t)
    assert np.array_equal(q1, q2) and np.array_equal(b1, b2)


def test_swiglu_requant_only():
    a, b, ref, G, D, Dq = _swiglu_case(256, 256, 256, seed=6, write_d=False)
    q_ref, s_ref, _ = o.requantize(ref, G)
    q, s, _, _ = read_nvfp4(Dq)
    # without the bf16 output to compare, the codes follow the oracle's up to one level and
    # one scale code, and differ on few elements
    assert np.all(np.abs(s.astype(int) - s_ref.astype(int)) <= 1)
    same = np.repeat(s == s_ref, 16, axis=1)
    assert np.all(np.abs(level_index(q) - level_index(q_ref))[same] <= 1)
    assert (q != q_ref).mean() < 0.01
    deq = o.dequantize(q, s, G)
    deq_ref = o.dequantize(q_ref, s_ref, G)
    assert np.linalg.norm(deq - deq_ref) / np.linalg.norm(deq_ref) < 1e-2


def test_unfused_ops_match_oracle():
    M, N, hd, nn = 256, 1024, 256, 768
    x = wk.activations(M, N, 0, seed=8)
    w = np.tile(wk.norm_weight(hd, 8), nn // hd).astype(np.float32)
    xd = x.to(device())
    y = xd.clone()
    ep.rmsnorm_heads_bf16(xd, torch.from_numpy(w).to(device()), hd, nn, 1e-6, y)
    ref = o.bf16_round(o.rmsnorm_heads(x.double().numpy(), w, hd, nn, 1e-6))
    assert_close(bf16_to_np(y), ref, "rmsnorm_heads_bf16")
    for hd2 in (128,):
        y2 = torch.empty_like(xd)
        w2 = np.tile(wk.norm_weight(hd2, 9), N // hd2).astype(np.float32)
        ep.rmsnorm_heads_bf16(xd, torch.from_numpy(w2).to(device()), hd2, N, 1e-6, y2)
        ref2 = o.bf16_round(o.rmsnorm_heads(x.double().numpy(), w2, hd2, N, 1e-6))
        assert_close(bf16_to_np(y2), ref2, "rmsnorm_heads_bf16 hd128")
    # a head count that is not a multiple of the kernel's heads per warp, computed in place
    xr = wk.activations(7, 768, 0, seed=11)
    wr = np.tile(wk.norm_weight(hd, 11), 3).astype(np.float32)
    yr = xr.to(device())
    ep.rmsnorm_heads_bf16(yr, torch.from_numpy(wr).to(device()), hd, 768, 1e-6, yr)
    refr = o.bf16_round(o.rmsnorm_heads(xr.double().numpy(), wr, hd, 768, 1e-6))
    assert_close(bf16_to_np(yr), refr, "rmsnorm_heads_bf16 ragged, in place")
    c = wk.activations(M, 2 * 512, 0, seed=10).to(device())
    ys = torch.empty(M, 512, dtype=torch.bfloat16, device=device())
    ep.swiglu_bf16(c, ys)
    refs = o.bf16_round(o.swiglu(c.double().cpu().numpy()))
    assert_close(bf16_to_np(ys), refs, "swiglu_bf16")


def test_bounded_wait_times_out_into_a_status_and_the_context_survives():
    assert ep.read_device_status() == 0
    ep.selftest_bounded_wait(2_000_000)  # 2 ms
    assert ep.read_device_status() == 6
    assert ep.read_device_status() == 0  # reading clears it
    # the context is still usable
    got, ref = _rmsnorm_case(128, 256, 256, 128, 256, seed=2)
    assert_close(got, ref, "after timeout")


def test_no_device_errors_recorded():
    torch.cuda.synchronize()
    assert ep.read_device_status() == 0


def test_rmsnorm_and_swiglu_respect_a_padded_output_pitch():
    """Outputs written into a wider buffer (leading dimension > N): the values match the
    contiguous results bit for bit and the columns past N stay untouched. M = 384 also puts
    the last pair tile half past M."""
    M, K, N, hd, nn = 384, 512, 768, 256, 512
    a = wk.activations(M, K, wk.outlier_count(K), seed=12)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=12)
    w = np.tile(wk.norm_weight(hd, 12), nn // hd).astype(np.float32)
    A, B = quantize_gpu(a), quantize_gpu(b)
    wt = torch.from_numpy(w).to(device())
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_rmsnorm(A, B, wt, hd, nn, 1e-6, D)
    Dp = torch.full((M, N + 64), 3.0, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_rmsnorm(A, B, wt, hd, nn, 1e-6, Dp[:, :N])
    assert torch.equal(Dp[:, :N], D)
    assert torch.all(Dp[:, N:] == 3.0)
    Bi = quantize_gpu(b, interleave=True)
    Y = torch.empty(M, N // 2, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_swiglu(A, Bi, Y, None)
    Yp = torch.full((M, N // 2 + 128), 3.0, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_swiglu(A, Bi, Yp[:, :N // 2], None)
    assert torch.equal(Yp[:, :N // 2], Y)
    assert torch.all(Yp[:, N // 2:] == 3.0)
