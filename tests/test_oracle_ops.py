"""Pins for the oracle's GEMM, per-head RMSNorm, SwiGLU and bf16 rounding (CPU only).

RMSNorm: y = x * rsqrt(mean(x^2) + eps) * weight over one head ("Serving sub-second
Ideogram v4 without quality loss", sections "Epilogue fusion in brief" and "Tiles and
fragments on Blackwell"). SwiGLU: SiLU(C[:, :N//2]) * C[:, N//2:] (section "Fusing
gated SiLU (SwiGLU)").
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o
import workloads as wk


def test_gemm_matches_triple_loop():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((5, 24))
    b = rng.standard_normal((7, 24))
    np.testing.assert_allclose(o.gemm(a, b), o.gemm_bruteforce(a, b), rtol=1e-13, atol=1e-13)


def test_gemm_on_decoded_nvfp4_is_exact_against_rational_arithmetic():
    M, N, K = 4, 3, 64
    qa = wk.fp4_codes_exact(M, K, 0, 11)
    qb = wk.fp4_codes_exact(N, K, 0, 12)
    sa = wk.pow2_scales_exact(M, K // 16, 0, 13)
    sb = wk.pow2_scales_exact(N, K // 16, 0, 14)
    sa_codes = o.e4m3_encode(sa.astype(np.float32))
    sb_codes = o.e4m3_encode(sb.astype(np.float32))
    A = o.dequantize(qa, sa_codes, 1.0)
    B = o.dequantize(qb, sb_codes, 1.0)
    C = o.gemm(A, B)
    lv = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
          Fraction(4), Fraction(6)]

    def val(code, scale):
        v = lv[int(code) & 7] * Fraction(scale)
        return -v if int(code) & 8 else v

    for m in range(M):
        for n in range(N):
            exact = sum(val(qa[m, k], sa[m, k // 16]) * val(qb[n, k], sb[n, k // 16])
                        for k in range(K))
            assert Fraction(C[m, n]) == exact


def test_rmsnorm_unit_rms_before_weight():
    rng = np.random.default_rng(2)
    for hd in (128, 256):
        x = rng.standard_normal((8, 4 * hd)) * 3.0
        y = o.rmsnorm_heads(x, np.ones(4 * hd), hd, 4 * hd, 0.0)
        rms = np.sqrt(np.mean(y.reshape(8, 4, hd) ** 2, axis=2))
        np.testing.assert_allclose(rms, 1.0, rtol=1e-12)
        eps = 0.5
        y = o.rmsnorm_heads(x, np.ones(4 * hd), hd, 4 * hd, eps)
        ms = np.mean(x.reshape(8, 4, hd) ** 2, axis=2)
        rms = np.sqrt(np.mean(y.reshape(8, 4, hd) ** 2, axis=2))
        np.testing.assert_allclose(rms, np.sqrt(ms / (ms + eps)), rtol=1e-12)


def test_rmsnorm_scale_invariance_and_head_independence():
    rng = np.random.default_rng(3)
    hd = 256
    x = rng.standard_normal((4, 3 * hd))
    w = 1 + 0.1 * rng.standard_normal(3 * hd)
    y = o.rmsnorm_heads(x, w, hd, 3 * hd, 0.0)
    np.testing.assert_allclose(o.rmsnorm_heads(7.5 * x, w, hd, 3 * hd, 0.0), y, rtol=1e-12)
    x2 = x.copy()
    x2[:, hd:2 * hd] *= -3.0
    x2[:, hd + 5] += 10
    y2 = o.rmsnorm_heads(x2, w, hd, 3 * hd, 0.0)
    assert np.array_equal(y2[:, :hd], y[:, :hd]) and np.array_equal(y2[:, 2 * hd:], y[:, 2 * hd:])
    assert not np.allclose(y2[:, hd:2 * hd], y[:, hd:2 * hd])


def test_rmsnorm_matches_torch_and_passes_v_through():
    rng = np.random.default_rng(4)
    hd, nn, n = 128, 512, 768
    x = rng.standard_normal((6, n)) * 2
    w = 1 + 0.1 * rng.standard_normal(nn)
    y = o.rmsnorm_heads(x, w, hd, nn, 1e-6)
    xt = torch.from_numpy(x[:, :nn].reshape(6, nn // hd, hd))
    wt = torch.from_numpy(w.reshape(nn // hd, hd))
    ref = torch.nn.functional.rms_norm(xt, (hd,), eps=1e-6) * wt
    np.testing.assert_allclose(y[:, :nn], ref.reshape(6, nn).numpy(), rtol=1e-12, atol=1e-14)
    assert np.array_equal(y[:, nn:], x[:, nn:])


def test_swiglu_matches_torch_and_gate_is_first_half():
    rng = np.random.default_rng(5)
    c = rng.standard_normal((5, 64)) * 4
    ref = torch.nn.functional.silu(torch.from_numpy(c[:, :32])) * torch.from_numpy(c[:, 32:])
    np.testing.assert_allclose(o.swiglu(c), ref.numpy(), rtol=1e-13, atol=1e-15)
    c[:, :32] = 0
    assert not o.swiglu(c).any()


def test_swiglu_interleaved_weight_gives_the_same_output():
    a = wk.activations(8, 64, 1, 0).float().numpy().astype(np.float64)
    b = wk.weights(32, 64, 0.1, 0).float().numpy().astype(np.float64)
    logical = o.swiglu(o.gemm(a, b))
    ci = o.gemm(a, o.interleave_gate_up(b))           # columns [g0, u0, g1, u1, ...]
    inter = o.silu(ci[:, 0::2]) * ci[:, 1::2]
    np.testing.assert_array_equal(inter, logical)


def test_bf16_round_matches_torch_cast_of_float32():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.standard_normal(100000) * 10 ** rng.uniform(-6, 6, 100000),
                        [0.0, -0.0, 1.0, 3.0 + 2 ** -8, 3.0 + 3 * 2 ** -8]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(o.bf16_round(x.astype(np.float64)), ref)


@pytest.mark.parametrize("M,N,K", [(8, 16, 64), (3, 5, 32)])
def test_problem_pipeline_small(M, N, K):
    a = wk.activations(M, K, 1, 0)
    b = wk.weights(N, K, 1 / np.sqrt(K), 0)
    c = o.problem_gemm(a, b)
    c_rows = o.problem_gemm(a, b, rows=np.array([1, 2]))
    np.testing.assert_array_equal(c[[1, 2]], c_rows)
    # FP4 GEMM is close to the bf16 GEMM at the FP4 error level
    ref = a.double().numpy() @ b.double().numpy().T
    rel = np.linalg.norm(c - ref) / np.linalg.norm(ref)
    assert rel < 0.3


def test_pointwise_matches_torch_float32_bias_add_and_relu():
    rng = np.random.default_rng(4)
    c = rng.standard_normal((64, 96)).astype(np.float32).astype(np.float64)  # float32-valued
    bias = (rng.standard_normal(96) * 3).astype(np.float32)
    got = o.pointwise(c, bias, relu=True)
    ref = torch.relu(torch.from_numpy(c.astype(np.float32)) + torch.from_numpy(bias)).double().numpy()
    assert np.array_equal(got, ref)
    # no bias, no activation: the float32 rounding of c only
    c2 = rng.standard_normal((8, 32))
    assert np.array_equal(o.pointwise(c2), c2.astype(np.float32).astype(np.float64))
    # ReLU zeroes exactly the negative sums
    y = o.pointwise(c, bias)
    assert np.array_equal(o.pointwise(c, bias, relu=True) == 0, y <= 0)


def _ab(M, N, K, seed):
    return wk.activations(M, K, 1, seed), wk.weights(N, K, 1 / np.sqrt(K), seed)


def test_problem_swiglu_is_odd_in_the_up_half_only():
    """silu(g) * u is odd in u and not in g. Quantisation is sign-symmetric (sign-magnitude
    codes, scales from |x|), so negating the up rows of B negates the output exactly, while
    negating the gate rows does not: a composition that swapped the halves fails."""
    M, Nh, K = 6, 32, 64
    a, b = _ab(M, 2 * Nh, K, 7)
    base = o.problem_swiglu(a, b)
    neg_up = torch.cat([b[:Nh], -b[Nh:]])
    np.testing.assert_array_equal(o.problem_swiglu(a, neg_up), -base)
    neg_gate = torch.cat([-b[:Nh], b[Nh:]])
    assert not np.array_equal(o.problem_swiglu(a, neg_gate), -base)
    assert base.shape == (M, Nh)


def test_problem_rmsnorm_is_invariant_to_a_power_of_two_scale_of_a():
    """Doubling A doubles G and leaves every code and block scale unchanged, so C doubles
    exactly. With eps = 0 the normalised heads do not move, and the passthrough (V) columns
    double exactly (bf16 rounding commutes with a power of two)."""
    M, N, K, hd = 4, 512, 256, 128
    a, b = _ab(M, N, K, 9)
    w = np.random.default_rng(1).uniform(0.5, 1.5, 256)
    y1 = o.problem_rmsnorm(a, b, w, hd, 256, 0.0)
    y2 = o.problem_rmsnorm(a * 2, b, w, hd, 256, 0.0)
    np.testing.assert_array_equal(y2[:, :256], y1[:, :256])
    np.testing.assert_array_equal(y2[:, 256:], 2 * y1[:, 256:])
    np.testing.assert_array_equal(y1[:, 256:], o.problem_plain(a, b)[:, 256:])


def test_problem_pointwise_relu_is_the_positive_part_of_the_same_sum():
    M, N, K = 5, 64, 128
    a, b = _ab(M, N, K, 11)
    bias = np.random.default_rng(2).standard_normal(N).astype(np.float32)
    y = o.problem_pointwise(a, b, bias)
    r = o.problem_pointwise(a, b, bias, relu=True)
    np.testing.assert_array_equal(r, np.maximum(y, 0.0))
    assert (y < 0).any() and (r >= 0).all()
