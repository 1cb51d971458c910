"""CPU oracle for the NVFP4 GEMM + fused-epilogue path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (the CUDA library and its binding) never calls it, and it shares no
code with that path.

It is the plain definition of what the path computes, written from
"Serving sub-second Ideogram v4 without quality loss" (fal):

* section "Running the transformer in FP4": an FP4 value has 1 sign, 2 exponent and
  1 mantissa bit (E2M1), and the matmul runs natively in 4 bits;
* section "Epilogue fusion in brief": the GEMM C = A @ B, then the small op; RMSNorm is
  y = x * rsqrt(mean(x^2) + eps) * weight, reduced over a whole head;
* section "Tiles and fragments on Blackwell": a head is head_dim (128 or 256) adjacent
  output columns;
* section "Fusing gated SiLU (SwiGLU)": output = SiLU(C[:, :N//2]) * C[:, N//2:], and
  the gate/up weight rows are interleaved once at packing time;
* section "Quantization-aware distillation": inference uses static FP4 quantisation.

The NVFP4 block format (16 elements along K share one unsigned E4M3 scale, one FP32
scale per tensor) is not spelled out on the page; the oracle uses that reading, with
the per-tensor scale G = amax / (6 * 448) so that the largest block scale lands on the
largest E4M3 value. Every quantisation decision (which code, which scale) is taken in
IEEE float32, in the exact operation order stated in ``quantize``; the GEMM,
normalisation and activation are evaluated in float64 on the decoded values and
rounded once to bfloat16 (round to nearest even).

Everything here is pinned by ``tests/test_oracle_*.py`` against closed forms, library
routines (torch's float8_e4m3fn cast, numpy matmul, torch rms_norm / silu), brute force
on tiny inputs and invariants; no function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

# ----------------------------------------------------------------------------------
# E2M1 (FP4) element codec: code bits  s e1 e0 m
# ----------------------------------------------------------------------------------

E2M1_MAX = 6.0


def e2m1_decode(codes) -> np.ndarray:
    """4-bit E2M1 codes (0..15) -> float64.

    e == 0 is subnormal: 0.5 * m; otherwise 2^(e-1) * (1 + m/2). The eight magnitudes
    are {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
    """
    c = np.asarray(codes).astype(np.int64) & 0xF
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(s == 1, -mag, mag)


_E2M1_MAGS = e2m1_decode(np.arange(8))          # increasing in the code
_E2M1_TABLE = e2m1_decode(np.arange(16))         # code -> value lookup


def _rne_to_table(ax: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of an increasing table, ties to the even index.

    ``ax`` is float64 (exact copies of float32 inputs); values above the last entry
    map to the last entry (saturation).
    """
    hi = np.searchsorted(table, ax, side="left")        # table[hi-1] < ax <= table[hi]
    hi = np.clip(hi, 1, len(table) - 1)
    lo = hi - 1
    dlo = ax - table[lo]
    dhi = table[hi] - ax
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(ax >= table[-1], len(table) - 1, idx)
    idx = np.where(ax <= table[0], 0, idx)
    return idx


def e2m1_encode(x) -> np.ndarray:
    """float32 -> E2M1 code, round to nearest with ties to the even mantissa,
    saturating at +-6. The sign bit follows the input's sign bit (so -0.1 -> 0x8).

    The magnitude index is the number of midpoints between adjacent levels that |x|
    lies above; at a midpoint exactly, the even index of the two neighbours wins.
    (Every midpoint is exact in float32, so the comparisons are exact.)
    """
    x = np.asarray(x, dtype=F32)
    ax = np.abs(x)
    idx = np.zeros(x.shape, np.uint8)
    for i in range(7):
        mid = F32((_E2M1_MAGS[i] + _E2M1_MAGS[i + 1]) / 2)
        idx += (ax > mid)
        if (i + 1) % 2 == 0:
            idx += (ax == mid)
    return idx | (np.signbit(x).astype(np.uint8) << 3)


# ----------------------------------------------------------------------------------
# E4M3 (unsigned use) block-scale codec: s eeee mmm, bias 7, 0x7F / 0xFF are NaN
# ----------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """8-bit E4M3 codes -> float64. e == 0: m/8 * 2^-6; else 2^(e-7) * (1 + m/8)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where(s == 1, -mag, mag)


_E4M3_MAGS = e4m3_decode(np.arange(0x7F))       # codes 0x00..0x7E, increasing
_E4M3_TABLE = e4m3_decode(np.arange(256))        # code -> value lookup


def e4m3_encode(x) -> np.ndarray:
    """Non-negative float32 -> E4M3 code, round to nearest even, saturating at 448."""
    ax = np.asarray(x, dtype=F32).astype(np.float64)
    if np.any(ax < 0) or np.any(np.isnan(ax)):
        raise ValueError("block scales are non-negative numbers")
    return _rne_to_table(ax, _E4M3_MAGS).astype(np.uint8)


# ----------------------------------------------------------------------------------
# NVFP4 block quantisation (16 elements along the contiguous axis share one scale)
# ----------------------------------------------------------------------------------

BLOCK = 16
GLOBAL_DIV = F32(6.0 * 448.0)    # amax / (largest E2M1 * largest E4M3)


def global_scale(x) -> np.float32:
    """Per-tensor FP32 scale G = amax(|x|) / 2688, computed in float32."""
    amax = F32(np.max(np.abs(np.asarray(x, dtype=F32)))) if np.size(x) else F32(0)
    return F32(amax / GLOBAL_DIV)


def quantize(x, G=None):
    """Quantise a (rows, cols) float32 tensor to NVFP4, blocks of 16 along cols.

    Steps, each an IEEE float32 operation in this order:
      G    = amax(|x|) / 2688                (unless a static G is given)
      enc  = 1 / (6 * G)
      per block of 16:  amax_b = max |x_i|
      s    = E4M3_rne_sat(amax_b * enc)     (s = 0 when amax_b == 0)
      d    = dec(s) * G
      r    = 1 / d
      q_i  = E2M1_rne_sat(x_i * r)          (q_i = 0 when d == 0)
    The decoded value of element i is dec(q_i) * dec(s) * G.

    Returns (codes uint8 (rows, cols), scales uint8 (rows, cols/16), G float32).
    """
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    if cols % BLOCK:
        raise ValueError("cols must be a multiple of 16")
    G = global_scale(x) if G is None else F32(G)
    blocks = x.reshape(rows, cols // BLOCK, BLOCK)
    amax_b = np.max(np.abs(blocks), axis=2) if cols else np.zeros((rows, 0), F32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        enc = F32(F32(1.0) / F32(F32(6.0) * G)) if G != 0 else F32(np.inf)
        sf = (amax_b * enc).astype(F32)
        sf = np.where(amax_b == 0, F32(0), sf)
        s = e4m3_encode(np.where(np.isinf(sf), F32(E4M3_MAX), sf))
        d = (e4m3_decode(s).astype(F32) * G).astype(F32)
        r = np.where(d > 0, F32(1.0) / np.where(d > 0, d, F32(1)), F32(0)).astype(F32)
        v = (blocks * r[:, :, None]).astype(F32)
    q = e2m1_encode(v)
    q = np.where((d > 0)[:, :, None], q, np.uint8(0)).astype(np.uint8)
    return q.reshape(rows, cols), s, G


def dequantize(codes, scales, G) -> np.ndarray:
    """dec(q) * dec(s) * G in float64, (rows, cols)."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    vals = _E2M1_TABLE[codes & 0xF].reshape(rows, cols // BLOCK, BLOCK)
    vals *= (_E4M3_TABLE[np.asarray(scales)] * float(G))[:, :, None]
    return vals.reshape(rows, cols)


def fake_quantize(x, G=None):
    """Quantise-dequantise ("fake quantisation" of quantisation-aware distillation, page
    "Serving sub-second Ideogram v4 without quality loss", section on quantization-aware
    distillation): the forward pass sees the FP4 rounding noise. Returns (y, G) with
    y = bf16(fp32(e2m1(q) * e4m3(s)) * fp32 G): the level-scale product is exact in fp32,
    the product with G is one fp32 rounding, the result is rounded to bf16 (RNE).
    The backward pass (straight-through estimator) is the identity and needs no oracle."""
    q, s, G = quantize(x, G)
    rows, cols = q.shape
    ls = (_E2M1_TABLE[q & 0xF].reshape(rows, cols // BLOCK, BLOCK)
          * _E4M3_TABLE[np.asarray(s)][:, :, None]).reshape(rows, cols)
    y32 = ls.astype(np.float32) * np.float32(G)
    return bf16_round(y32.astype(np.float64)), G


# ----------------------------------------------------------------------------------
# Storage layouts read by the tensor cores (an independent statement of the byte
# layout, used to read GPU buffers and to build GPU inputs in tests)
# ----------------------------------------------------------------------------------

def pack_codes(codes) -> np.ndarray:
    """(rows, cols) codes -> (rows, cols/2) bytes; element 2j in bits 0-3 of byte j,
    element 2j+1 in bits 4-7."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def sf_bytes(rows: int, cols: int) -> int:
    """Size of the block-scale buffer: rows padded to 128, 16-blocks padded to 4."""
    return ((rows + 127) // 128) * 128 * ((cols // BLOCK + 3) // 4) * 4


def sf_offset(row, kb, cols: int):
    """Byte offset of the scale of (row, 16-block kb) in the tensor-core scale layout.

    The scales of a 128-row x 4-block tile form one 512-byte unit; units are ordered
    row-tile major, then 4-block group. Inside a unit, row r and block c sit at
    (r % 32) * 16 + (r // 32) * 4 + c: 32 lines of 16 bytes, each line holding rows
    r, r+32, r+64, r+96.
    """
    row = np.asarray(row)
    kb = np.asarray(kb)
    groups = (cols // BLOCK + 3) // 4
    unit = (row // 128) * groups + kb // 4
    r = row % 128
    return unit * 512 + (r % 32) * 16 + (r // 32) * 4 + kb % 4


def pack_scales(scales, cols: int) -> np.ndarray:
    """(rows, cols/16) scale codes -> flat layout buffer (padding bytes are 0)."""
    s = np.asarray(scales, dtype=np.uint8)
    rows, nkb = s.shape
    buf = np.zeros(sf_bytes(rows, cols), np.uint8)
    rr, kk = np.meshgrid(np.arange(rows), np.arange(nkb), indexing="ij")
    buf[sf_offset(rr, kk, cols)] = s
    return buf


def unpack_scales(buf, rows: int, cols: int) -> np.ndarray:
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    rr, kk = np.meshgrid(np.arange(rows), np.arange(cols // BLOCK), indexing="ij")
    return buf[sf_offset(rr, kk, cols)]


def interleave_gate_up(rows_gate_up) -> np.ndarray:
    """Pack-time permutation of a [gate | up] weight (2*Nh rows) into
    [gate0, up0, gate1, up1, ...]: packed row 2j = gate row j, 2j+1 = up row j."""
    w = np.asarray(rows_gate_up)
    nh = w.shape[0] // 2
    out = np.empty_like(w)
    out[0::2] = w[:nh]
    out[1::2] = w[nh:]
    return out


# ----------------------------------------------------------------------------------
# GEMM and the fused ops, in float64
# ----------------------------------------------------------------------------------

def gemm(a_dec, b_dec) -> np.ndarray:
    """C[m, n] = sum_k A[m, k] * B[n, k], float64 (B stored N x K)."""
    return np.asarray(a_dec, np.float64) @ np.asarray(b_dec, np.float64).T


def gemm_bruteforce(a_dec, b_dec) -> np.ndarray:
    """Triple loop, for tiny shapes only."""
    a = np.asarray(a_dec, np.float64)
    b = np.asarray(b_dec, np.float64)
    M, K = a.shape
    N = b.shape[0]
    c = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += a[m, k] * b[n, k]
            c[m, n] = acc
    return c


def rmsnorm_heads(x, w, head_dim: int, n_norm_cols: int, eps: float) -> np.ndarray:
    """Per row and per head of head_dim adjacent columns among the first n_norm_cols:
    y = x * rsqrt(mean(x^2) + eps) * w[col]; the remaining columns pass through."""
    x = np.asarray(x, np.float64)
    y = x.copy()
    M = x.shape[0]
    heads = x[:, :n_norm_cols].reshape(M, n_norm_cols // head_dim, head_dim)
    ms = np.mean(heads * heads, axis=2, keepdims=True)
    normed = heads / np.sqrt(ms + eps)
    y[:, :n_norm_cols] = normed.reshape(M, n_norm_cols) * np.asarray(w, np.float64)[None, :]
    return y


def pointwise(c, bias=None, relu: bool = False) -> np.ndarray:
    """Pointwise epilogue of page "Serving sub-second Ideogram v4 without quality loss",
    section "Epilogue fusion in brief" (bias, ReLU, cast): y = act(c + bias[n]) for an
    alpha-scaled accumulator c. The sum is rounded once to float32 (the GPU forms
    alpha * acc + bias with one fused multiply-add); returned as float64 holding float32
    values, ready for the cast (bf16_round, or numpy's float16/float32)."""
    y = np.asarray(c, np.float64)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    y = y.astype(F32).astype(np.float64)
    if relu:
        y = np.maximum(y, 0.0)
    return y


def silu(x) -> np.ndarray:
    x = np.asarray(x, np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def swiglu(c) -> np.ndarray:
    """output = SiLU(C[:, :N//2]) * C[:, N//2:] (gate = first half)."""
    c = np.asarray(c, np.float64)
    nh = c.shape[1] // 2
    return silu(c[:, :nh]) * c[:, nh:]


def bf16_round(x) -> np.ndarray:
    """float64 -> nearest bfloat16 value (ties to even), returned as float64."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def bf16_bits(x) -> np.ndarray:
    """bfloat16-valued float64 -> uint16 bit patterns."""
    f = np.asarray(x, np.float64).astype(F32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------------
# Whole problems: bf16 inputs -> quantise -> GEMM -> op -> bf16 (-> NVFP4)
# ----------------------------------------------------------------------------------

def _as_f32(t) -> np.ndarray:
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.float().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, F32)


def quantized_operand(x_bf16):
    """Quantise a bf16 operand with its own amax-derived G. Returns (codes, scales, G)."""
    return quantize(_as_f32(x_bf16))


def problem_gemm(a_bf16, b_bf16, rows=None, b_quant=None) -> np.ndarray:
    """float64 C = dequant(A) @ dequant(B)^T.

    rows: optionally only these rows of A. Quantisation is row-local once G is fixed,
    so the rows are quantised with the whole tensor's G (identical to quantising all of
    A and keeping those rows).
    b_quant: optionally the (codes, scales, G) of B from an earlier quantized_operand(b).
    """
    a = _as_f32(a_bf16)
    Ga = global_scale(a)
    if rows is not None:
        a = a[np.asarray(rows)]
    qa, sa, _ = quantize(a, Ga)
    qb, sb, gb = quantized_operand(b_bf16) if b_quant is None else b_quant
    return gemm(dequantize(qa, sa, Ga), dequantize(qb, sb, gb))


def problem_plain(a_bf16, b_bf16, rows=None, b_quant=None) -> np.ndarray:
    return bf16_round(problem_gemm(a_bf16, b_bf16, rows, b_quant))


def problem_rmsnorm(a_bf16, b_bf16, w, head_dim, n_norm_cols, eps, rows=None, b_quant=None) -> np.ndarray:
    c = problem_gemm(a_bf16, b_bf16, rows, b_quant)
    return bf16_round(rmsnorm_heads(c, w, head_dim, n_norm_cols, eps))


def problem_pointwise(a_bf16, b_bf16, bias=None, relu=False, rows=None, b_quant=None) -> np.ndarray:
    return pointwise(problem_gemm(a_bf16, b_bf16, rows, b_quant), bias, relu)


def problem_swiglu(a_bf16, b_gate_up_bf16, rows=None, b_quant=None) -> np.ndarray:
    """b_gate_up is the logical [gate | up] weight (2*Nh x K)."""
    return bf16_round(swiglu(problem_gemm(a_bf16, b_gate_up_bf16, rows, b_quant)))


def requantize(out_bf16_values, G):
    """Static-scale NVFP4 quantisation of bf16-valued outputs (blocks along N)."""
    return quantize(np.asarray(out_bf16_values, np.float64).astype(F32), G)


# ----------------------------------------------------------------------------------
# MXFP4 with a block-local transform (page "KroQuant: efficient post-training
# quantization for diffusion transformers via Kronecker-product structure": activations
# split into independent blocks of 32, each with an invertible Kronecker-structured
# transform; MXFP4 format). The pages' transforms are learned; this build uses a fixed
# one, the 32-point Walsh-Hadamard matrix H_2 (x) H_2 (x) H_2 (x) H_2 (x) H_2.
# MXFP4 per the OCP Microscaling format: E2M1 elements, one E8M0 (power-of-two) scale
# per 32 elements, no per-tensor scale.
# ----------------------------------------------------------------------------------

MX_BLOCK = 32


def e8m0_decode(codes) -> np.ndarray:
    """E8M0 scale code e -> 2^(e - 127) (float64; code 255 is NaN and never produced)."""
    e = np.asarray(codes, dtype=np.int64)
    return np.ldexp(1.0, e - 127)


def mx_quantize(x):
    """Quantise (rows, cols) float32 to MXFP4, blocks of 32 along cols. Per block: the
    shared exponent is floor(log2(amax)) - 2 (2 = the exponent of E2M1's largest value,
    6 = 1.5 * 2^2), clamped to [-127, 127]; the scale is X = 2^that; elements are
    E2M1_rn_satfinite(x / X) (x / X is exact: X is a power of two). An all-zero block gets
    code 0 and zero elements. Returns (codes (rows, cols) uint8, e8m0 (rows, cols/32))."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    xb = x.reshape(rows, cols // MX_BLOCK, MX_BLOCK).astype(np.float64)
    amax = np.abs(xb).max(axis=2)
    _, p = np.frexp(amax)                      # amax = m * 2^p, 0.5 <= m < 1
    shared = np.clip(p - 1 - 2, -127, 127)     # floor(log2 amax) - 2
    e = np.where(amax > 0, shared + 127, 0).astype(np.uint8)
    X = np.ldexp(1.0, shared)[:, :, None]
    q = e2m1_encode((xb / X).astype(F32).reshape(rows, cols))
    q = np.where(np.repeat(amax > 0, MX_BLOCK, axis=1), q, 0).astype(np.uint8)
    return q, e


def mx_dequantize(codes, e8m0) -> np.ndarray:
    """dec(q) * 2^(e - 127) in float64, (rows, cols)."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    vals = _E2M1_TABLE[codes & 0xF].reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    vals *= e8m0_decode(e8m0)[:, :, None]
    return vals.reshape(rows, cols)


def hadamard32(x) -> np.ndarray:
    """x @ H32 per block of 32 along cols, H32 the unnormalised Sylvester-Hadamard matrix
    (entries +-1), computed in float32 by the fast Walsh-Hadamard transform: five stages,
    stage h in (1, 2, 4, 8, 16) maps each pair (j, j + h), j with bit h clear, to
    (a + b, a - b). H32 H32^T = 32 I, so (x H)(w H)^T = 32 x w^T."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    y = x.reshape(rows, cols // MX_BLOCK, MX_BLOCK).copy()
    h = 1
    while h < MX_BLOCK:
        y = y.reshape(rows, cols // MX_BLOCK, MX_BLOCK // (2 * h), 2, h)
        a, b = y[:, :, :, 0, :].copy(), y[:, :, :, 1, :].copy()
        y[:, :, :, 0, :] = a + b
        y[:, :, :, 1, :] = a - b
        h *= 2
    return y.reshape(rows, cols)


def mx_sf_bytes(rows: int, cols: int) -> int:
    """Size of an MXFP4 scale buffer: the tensor-core scale layout with 32-blocks (a
    512-byte unit holds 128 rows x 4 blocks, i.e. 128 K values)."""
    return sf_bytes(rows, cols // 2)


def mx_pack_scales(e8m0, cols: int) -> np.ndarray:
    """(rows, cols/32) E8M0 codes -> flat layout buffer: the same unit layout as
    pack_scales, counting blocks of 32 (so it is pack_scales at half the columns)."""
    return pack_scales(e8m0, cols // 2)


def mx_unpack_scales(buf, rows: int, cols: int) -> np.ndarray:
    return unpack_scales(buf, rows, cols // 2)
