"""GPU parity of the MXFP4 path: mxfp4_quantize without the transform bit for bit against
the oracle; with the 32-point block Hadamard transform, equal to the plain definition
(x H32 exactly, rounded once to float32, then MXFP4) except where the float32 error of
evaluating the transform decides a rounding, and bit for bit equal to the oracle's float32
butterfly order; the MXFP4 GEMM exact on exactly
representable operands (pins the E8M0 scale layout and the block32 MMA descriptor), and
within tolerance on workload operands; the transform lowers the error on outlier
channels, which is its purpose."""
import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_close, bf16_bits, device

pytestmark = pytest.mark.gpu


def _read_mx(t):
    torch.cuda.synchronize()
    q = o.unpack_codes(t.codes.cpu().numpy())
    buf = t.sf.cpu().numpy()
    e = o.mx_unpack_scales(buf, t.rows, t.cols)
    return q, e, float(t.gscale.item()), buf


@pytest.mark.parametrize("rows,cols", [(256, 1024), (130, 384), (4096, 3072), (1, 128)])
@pytest.mark.parametrize("hadamard", [False, True])
def test_mx_quantize_matches_oracle_bitwise(rows, cols, hadamard):
    x = wk.activations(rows, cols, 3, seed=rows + cols)
    t = ep.mxfp4_quantize(x.to(device()), ep.NVFP4Tensor.empty_mx(rows, cols, device()), hadamard=hadamard)
    xf = x.float().numpy()
    q, e, g, buf = _read_mx(t)
    if hadamard:
        _check_transform_plain(q, e, xf)
    q_ref, e_ref = o.mx_quantize(o.hadamard32_fp32_order(xf) if hadamard else xf)
    assert np.array_equal(e, e_ref), f"{int((e != e_ref).sum())} scale mismatches"
    assert np.array_equal(q, q_ref), f"{int((q != q_ref).sum())} code mismatches"
    assert np.array_equal(buf, o.mx_pack_scales(e_ref, cols))  # padding bytes are 0
    assert g == (float(np.float32(1 / np.sqrt(32))) if hadamard else 1.0)


@pytest.mark.parametrize("hadamard", [False, True])
def test_mx_quantize_off_a_32_byte_boundary_and_strided(hadamard):
    """x starting 16 bytes past a 32-byte boundary (128-bit loads) and x with a row pitch
    above cols: the same codes and scales as the oracle."""
    rows, cols = 260, 512
    x = wk.activations(rows, cols, 3, seed=17)
    flat = torch.empty(rows * cols + 8, dtype=torch.bfloat16, device=device())
    xo = flat[8:].view(rows, cols)
    assert xo.data_ptr() % 32 == 16
    xo.copy_(x.to(device()))
    big = torch.zeros(rows, cols + 136, dtype=torch.bfloat16, device=device())
    xs = big[:, 8:8 + cols]
    xs.copy_(x.to(device()))
    q_ref, e_ref = o.mx_quantize(o.hadamard32_fp32_order(x.float().numpy()) if hadamard else x.float().numpy())
    for xin in (xo, xs):
        t = ep.mxfp4_quantize(xin, ep.NVFP4Tensor.empty_mx(rows, cols, device()), hadamard=hadamard)
        q, e, _, buf = _read_mx(t)
        assert np.array_equal(e, e_ref) and np.array_equal(q, q_ref)
        assert np.array_equal(buf, o.mx_pack_scales(e_ref, cols))


def _check_transform_plain(q, e, xf):
    """Codes and E8M0 scales of the transformed tensor against the plain definition
    mx_quantize(hadamard32(x)): a scale may differ only in a block whose amax is within
    the transform's float32 error band of a power of two; codes only at element ties, or,
    in a block whose scale took the other side, they are the plain rounding under the GPU's
    scale."""
    q_ref, e_ref = o.mx_quantize(o.hadamard32(xf))
    bt, et = o.mx_transform_ties(xf)
    ed = e != e_ref
    assert not (ed & ~bt).any(), f"{int((ed & ~bt).sum())} scales differ outside a tie"
    same = np.repeat(~ed, 32, axis=1)
    assert not ((q != q_ref) & same & ~et).any(), "codes differ outside a tie"
    if ed.any():
        q_alt = o.mx_codes_for_scales(o.hadamard32(xf), e)
        _, et_alt = o.mx_transform_ties(xf, e)
        assert not ((q != q_alt) & ~same & ~et_alt).any(), "codes under a tie scale differ outside a tie"


def _mx_from_arrays(codes, e8m0, g=1.0):
    rows, cols = codes.shape
    t = ep.NVFP4Tensor.empty_mx(rows, cols, device())
    t.codes.copy_(torch.from_numpy(o.pack_codes(codes)))
    t.sf.copy_(torch.from_numpy(o.mx_pack_scales(e8m0, cols)))
    t.gscale.fill_(g)
    return t


def _exact(M, N, K, seed):
    qa, qb = wk.fp4_codes_exact(M, K, seed, 41), wk.fp4_codes_exact(N, K, seed, 42)
    ea = (127 + np.log2(wk.pow2_scales_exact(M, K // 32, seed, 43))).astype(np.uint8)
    eb = (127 + np.log2(wk.pow2_scales_exact(N, K // 32, seed, 44))).astype(np.uint8)
    return qa, ea, qb, eb


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (384, 768, 3072), (2048, 2560, 256)])
def test_mx_gemm_is_exact_on_exactly_representable_inputs(M, N, K):
    qa, ea, qb, eb = _exact(M, N, K, seed=M + N + K)
    A, B = _mx_from_arrays(qa, ea), _mx_from_arrays(qb, eb, 0.5)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_mxfp4_plain(A, B, D)
    ref = o.bf16_round(0.5 * o.gemm(o.mx_dequantize(qa, ea), o.mx_dequantize(qb, eb)))
    got, want = bf16_bits(D), o.bf16_bits(ref)
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} outputs differ"


def test_mx_gemm_pointwise_f32_bias_relu_exact():
    M, N, K = 256, 512, 512
    qa, ea, qb, eb = _exact(M, N, K, seed=9)
    A, B = _mx_from_arrays(qa, ea), _mx_from_arrays(qb, eb)
    bias = (np.random.default_rng(5).standard_normal(N)).astype(np.float32)
    D = torch.empty(M, N, dtype=torch.float32, device=device())
    ep.gemm_mxfp4_pointwise(A, B, D, bias=torch.from_numpy(bias).to(device()), relu=True)
    want = o.pointwise(o.gemm(o.mx_dequantize(qa, ea), o.mx_dequantize(qb, eb)), bias, relu=True).astype(np.float32)
    assert np.array_equal(D.cpu().numpy(), want)


@pytest.mark.parametrize("M", [256, 384])
def test_mx_gemm_with_transform_matches_oracle_and_beats_no_transform_on_outliers(M):
    K, N = 1024, 512
    a = wk.activations(M, K, 8, seed=M)       # 8 outlier channels x20
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=M + 1)
    errs = {}
    for hadamard in (False, True):
        A = ep.mxfp4_quantize(a.to(device()), ep.NVFP4Tensor.empty_mx(M, K, device()), hadamard=hadamard)
        B = ep.mxfp4_quantize(b.to(device()), ep.NVFP4Tensor.empty_mx(N, K, device()), hadamard=hadamard)
        D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
        ep.gemm_mxfp4_plain(A, B, D)
        af, bf = a.float().numpy(), b.float().numpy()
        if hadamard:
            af, bf = o.hadamard32(af), o.hadamard32(bf)
        g = float(np.float32(1 / np.sqrt(32))) if hadamard else 1.0
        ref = o.bf16_round(g * g * o.gemm(o.mx_dequantize(*o.mx_quantize(af)), o.mx_dequantize(*o.mx_quantize(bf))))
        got = D.float().cpu().numpy().astype(np.float64)
        assert_close(got, ref, f"mxfp4 gemm hadamard={hadamard}")
        exact = a.double().numpy() @ b.double().numpy().T
        errs[hadamard] = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert errs[True] < errs[False], errs
    assert ep.read_device_status() == 0


def test_mx_quantize_interleaved_weight_bitwise():
    w = wk.weights(2 * 200, 256, 1 / 16, seed=21)
    t = ep.mxfp4_quantize(w.to(device()), ep.NVFP4Tensor.empty_mx(400, 256, device()), hadamard=True, interleave=True)
    wi = o.interleave_gate_up(w.float().numpy())
    q, e, _, _ = _read_mx(t)
    _check_transform_plain(q, e, wi)
    q_ref, e_ref = o.mx_quantize(o.hadamard32_fp32_order(wi))
    assert np.array_equal(e, e_ref) and np.array_equal(q, q_ref)


@pytest.mark.parametrize("M,hd", [(256, 256), (384, 128)])
def test_mx_rmsnorm_gemm_matches_oracle(M, hd):
    K, N, n_norm = 1024, 1024, 512
    a = wk.activations(M, K, 2, seed=M)
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=M + 1)
    w = np.tile(wk.norm_weight(hd, 0, 3), n_norm // hd).astype(np.float32)
    A = ep.mxfp4_quantize(a.to(device()), ep.NVFP4Tensor.empty_mx(M, K, device()), hadamard=True)
    B = ep.mxfp4_quantize(b.to(device()), ep.NVFP4Tensor.empty_mx(N, K, device()), hadamard=True)
    D = torch.empty(M, N, dtype=torch.bfloat16, device=device())
    ep.gemm_mxfp4_rmsnorm(A, B, torch.from_numpy(w).to(device()), hd, n_norm, 1e-6, D)
    g = float(np.float32(1 / np.sqrt(32)))
    c = g * g * o.gemm(o.mx_dequantize(*o.mx_quantize(o.hadamard32(a.float().numpy()))),
                       o.mx_dequantize(*o.mx_quantize(o.hadamard32(b.float().numpy()))))
    ref = o.bf16_round(o.rmsnorm_heads(c, w, hd, n_norm, 1e-6))
    assert_close(D.float().cpu().numpy().astype(np.float64), ref, "mxfp4 rmsnorm")


def test_mx_swiglu_gemm_matches_oracle():
    M, K, nh = 256, 512, 512
    a = wk.activations(M, K, 2, seed=3)
    b = wk.weights(2 * nh, K, 1 / np.sqrt(K), seed=4)
    A = ep.mxfp4_quantize(a.to(device()), ep.NVFP4Tensor.empty_mx(M, K, device()), hadamard=True)
    B = ep.mxfp4_quantize(b.to(device()), ep.NVFP4Tensor.empty_mx(2 * nh, K, device()), hadamard=True, interleave=True)
    D = torch.empty(M, nh, dtype=torch.bfloat16, device=device())
    ep.gemm_mxfp4_swiglu(A, B, D)
    g = float(np.float32(1 / np.sqrt(32)))
    c = g * g * o.gemm(o.mx_dequantize(*o.mx_quantize(o.hadamard32(a.float().numpy()))),
                       o.mx_dequantize(*o.mx_quantize(o.hadamard32(b.float().numpy()))))
    ref = o.bf16_round(o.swiglu(c))
    assert_close(D.float().cpu().numpy().astype(np.float64), ref, "mxfp4 swiglu")
    assert ep.read_device_status() == 0
