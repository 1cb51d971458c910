"""GPU parity on the full-size workloads: the tiny QK-norm case, the SwiGLU case, the
1K-image QKV and FFN blocks, and the sweep over M in {1024, 4096, 8192, 16384} for QKV
(head_dim 128 and 256) and FFN-up (SwiGLU + NVFP4 re-quantisation). The GPU computes the
whole problem in the launch configuration bench.py uses. The oracle computes every row up
to M = 4096 (and every row of the largest problem, FFN-up at M = 16384, in row chunks);
above that a seeded sample of at least 2048 rows x all columns: the first and last rows,
one row in every 256-row band (so every tile row of the pair kernel is seen) and random
rows. Re-quantised codes follow the quantised-output rule (re-quantisation of the GPU's
own bf16 output up to ties; against the oracle's codes a differing code or scale only
where the bf16 values differ, by one level or one scale code)."""
import functools

import numpy as np
import pytest
import torch

import epilogues_nvfp4_quantize_b200 as ep
from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_close, assert_close_chain, assert_requant_point13, bf16_to_np, device, quantize_gpu, read_nvfp4

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=8)
def _weights(N, K, seed, interleave):
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=seed)
    return b, quantize_gpu(b, interleave=interleave)


@functools.lru_cache(maxsize=8)
def _oracle_b(N, K, seed):
    b = wk.weights(N, K, 1 / np.sqrt(K), seed=seed)
    return o.quantized_operand(b)


SAMPLE_ROWS = 2048


def _rows(M, n, seed=0):
    """None (all rows), or at least n seeded rows: first, last, one per 256-row band, and
    random rows."""
    if n is None or n >= M:
        return None
    rng = np.random.default_rng([seed, M])
    bands = np.arange(0, M, 256)
    per_band = bands + rng.integers(0, np.minimum(256, M - bands))
    extra = rng.choice(np.arange(M), size=n, replace=False)
    return np.unique(np.concatenate([[0, M - 1], per_band, extra]))


def _run_rmsnorm(wl, sample):
    a = wk.activations(wl.M, wl.K, wl.outliers, wl.seed)
    b, B = _weights(wl.N, wl.K, wl.seed, False)
    w = wk.norm_weight_columns(wl)
    A = quantize_gpu(a)
    D = torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_rmsnorm(A, B, torch.from_numpy(w).to(device()), wl.head_dim, wl.n_norm_cols, wl.eps, D)
    rows = _rows(wl.M, sample)
    ref = o.problem_rmsnorm(a, b, w, wl.head_dim, wl.n_norm_cols, wl.eps, rows=rows,
                            b_quant=_oracle_b(wl.N, wl.K, wl.seed))
    got = bf16_to_np(D) if rows is None else bf16_to_np(D[torch.from_numpy(rows).to(device())])
    return assert_close(got, ref, wl.name)


def _run_swiglu(wl, sample, requant=True):
    a = wk.activations(wl.M, wl.K, wl.outliers, wl.seed)
    b, B = _weights(wl.N, wl.K, wl.seed, True)
    A = quantize_gpu(a)
    nh = wl.N // 2
    rows = _rows(wl.M, sample)
    ref = o.problem_swiglu(a, b, rows=rows, b_quant=_oracle_b(wl.N, wl.K, wl.seed))
    G = np.float32(np.abs(ref).max() / 2688)
    D = torch.empty(wl.M, nh, dtype=torch.bfloat16, device=device())
    Dq = None
    if requant:
        Dq = ep.NVFP4Tensor.empty(wl.M, nh, device())
        Dq.gscale.fill_(float(G))
    ep.gemm_nvfp4_swiglu(A, B, D, Dq)
    sel = None if rows is None else torch.from_numpy(rows).to(device())
    got = bf16_to_np(D) if sel is None else bf16_to_np(D[sel])
    res = assert_close(got, ref, wl.name)
    if requant:
        q, s, _, _ = read_nvfp4(Dq)
        if rows is not None:
            q, s = q[rows], s[rows]
        share = assert_requant_point13(q, s, got, ref, G, wl.name + " requant")
        assert share < 0.01
    return res, (A, D, Dq, G, rows, ref)


def test_tiny_qk_norm():
    _run_rmsnorm(wk.qk_norm_tiny(), None)


def test_swiglu_1024():
    _run_swiglu(wk.swiglu_1024(), None, requant=False)


def test_qkv_1k_image():
    _run_rmsnorm(wk.qkv(4096, 256), None)


def test_ffn_block_1k_image_up_then_down():
    up = wk.ffn_up(4096, True)
    (_, (A, D, Dq, G, rows, h_ref)) = _run_swiglu(up, SAMPLE_ROWS)
    down = wk.ffn_down(4096)
    bd, Bd = _weights(down.N, down.K, down.seed, False)
    out = torch.empty(down.M, down.N, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_plain(Dq, Bd, out)
    # oracle chain on the same rows: its own bf16 FFN-up output, re-quantised with the same
    # static scale, then the down GEMM
    qh, sh, _ = o.requantize(h_ref, G)
    qb, sb, gb = _oracle_b(down.N, down.K, down.seed)
    ref = o.bf16_round(o.gemm(o.dequantize(qh, sh, G), o.dequantize(qb, sb, gb)))
    assert_close_chain(bf16_to_np(out[torch.from_numpy(rows).to(device())]), ref, "ffn_down")


@pytest.mark.parametrize("M", wk.SWEEP_M)
@pytest.mark.parametrize("kind", ["qkv_hd128", "qkv_hd256", "ffn_up"])
def test_sweep(M, kind):
    sample = None if M <= 4096 else SAMPLE_ROWS
    if kind == "ffn_up":
        _run_swiglu(wk.ffn_up(M, True), sample)
    else:
        _run_rmsnorm(wk.qkv(M, 128 if kind == "qkv_hd128" else 256), sample)


def test_ffn_up_16384_every_row():
    """The largest problem (the bench's FFN-up GEMM, M = 16384, N = 24576, K = 3072) with
    every output row compared against the oracle, in chunks of 2048 rows."""
    wl = wk.ffn_up(16384, True)
    a = wk.activations(wl.M, wl.K, wl.outliers, wl.seed)
    b, B = _weights(wl.N, wl.K, wl.seed, True)
    A = quantize_gpu(a)
    nh = wl.N // 2
    D = torch.empty(wl.M, nh, dtype=torch.bfloat16, device=device())
    ep.gemm_nvfp4_swiglu(A, B, D, None)
    torch.cuda.synchronize()
    bq = _oracle_b(wl.N, wl.K, wl.seed)
    worst = 0.0
    for r0 in range(0, wl.M, 2048):
        rows = np.arange(r0, r0 + 2048)
        ref = o.problem_swiglu(a, b, rows=rows, b_quant=bq)
        got = bf16_to_np(D[r0:r0 + 2048])
        worst = max(worst, assert_close(got, ref, f"{wl.name} rows {r0}..{r0 + 2047}")[0])
    assert ep.read_device_status() == 0


def test_no_device_errors_recorded():
    assert ep.read_device_status() == 0
