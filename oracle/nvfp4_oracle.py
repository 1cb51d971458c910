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
the per-tensor scale G = amax / (6 * 448) (an FP32 number) so that the largest block
scale lands on the largest E4M3 value.

Two statements of the quantiser live here:

* ``quantize`` is the plain definition: the block scale is the E4M3 value nearest to
  amax_b / (6 G) and each code the E2M1 value nearest to x / d, both decided on the exact
  quotients (ties to the even code). It is the oracle's answer.
* ``quantize_fp32_order`` takes the same decisions through IEEE float32 reciprocals and
  products, the order a GPU evaluates cheaply. Its results differ from the plain
  definition only where a quotient lies within ``TIE_REL`` of a rounding midpoint;
  ``quantize_ties`` marks those places. Tests compare a GPU result with the plain
  definition (codes and scales may differ only at those ties) and, bit for bit, with the
  float32 order.

The GEMM, normalisation and activation are evaluated in float64 on the decoded values and
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
    """Real number (float32 or float64) -> E2M1 code, round to nearest with ties to the
    even mantissa, saturating at +-6. The sign bit follows the input's sign bit (so
    -0.1 -> 0x8).

    The magnitude index is the number of midpoints between adjacent levels that |x|
    lies above; at a midpoint exactly, the even index of the two neighbours wins.
    (Every midpoint is exact in binary floating point, so the comparisons are exact.)
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    idx = np.zeros(x.shape, np.uint8)
    for i in range(7):
        mid = (_E2M1_MAGS[i] + _E2M1_MAGS[i + 1]) / 2
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
    """Non-negative real number (float32 or float64) -> E4M3 code, round to nearest
    even, saturating at 448 (infinity saturates too)."""
    ax = np.asarray(x, dtype=np.float64)
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


def _blocks(x):
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    if cols % BLOCK:
        raise ValueError("cols must be a multiple of 16")
    return x, x.reshape(rows, cols // BLOCK, BLOCK)


def quantize(x, G=None):
    """Quantise a (rows, cols) float32 tensor to NVFP4, blocks of 16 along cols: the plain
    definition.

      G    = fp32(amax(|x|) / 2688)           (unless a static G is given)
      per block of 16:  amax_b = max |x_i|
      s    = E4M3_rne_sat(amax_b / (6 G))     (0 when amax_b == 0)
      d    = dec(s) * G
      q_i  = E2M1_rne_sat(x_i / d)            (0 when d == 0)

    The decoded value of element i is dec(q_i) * dec(s) * G.

    Both roundings are decided on the exact quotient. The quotients are formed in float64,
    which decides them exactly: d has at most 28 significant bits (4 of dec(s), 24 of G)
    and 6 G at most 26, so a float32 numerator is either exactly on a rounding midpoint
    (at most 5 significant bits) times the denominator, or at least 2^-31 (relative) away
    from it, far more than float64's 2^-53 rounding of the quotient. dec(s) * G is exact
    in float64.

    Returns (codes uint8 (rows, cols), scales uint8 (rows, cols/16), G float32).
    """
    x, blocks = _blocks(x)
    rows, cols = x.shape
    G = global_scale(x) if G is None else F32(G)
    amax_b = np.max(np.abs(blocks), axis=2).astype(np.float64) if cols else np.zeros((rows, 0))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(amax_b > 0, amax_b / (6.0 * float(G)), 0.0)   # +inf when G == 0
    s = e4m3_encode(ratio)
    return codes_for_scales(x, s, G), s, G


def _quotients(x, s, G):
    """x_i / d per element (float64) and d > 0 per block, d = dec(s) * G (exact)."""
    x, blocks = _blocks(x)
    d = e4m3_decode(s) * float(G)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = blocks.astype(np.float64) / np.where(d > 0, d, 1.0)[:, :, None]
    return v, d > 0


def codes_for_scales(x, s, G) -> np.ndarray:
    """The element step of ``quantize`` for given block scale codes s:
    q_i = E2M1_rne_sat(x_i / (dec(s) * G)), 0 where that scale is 0."""
    v, pos = _quotients(x, s, G)
    q = np.where(pos[:, :, None], e2m1_encode(v), np.uint8(0)).astype(np.uint8)
    return q.reshape(np.shape(x))


def code_ties_for_scales(x, s, G) -> np.ndarray:
    """Elements whose quotient x_i / (dec(s) * G) lies within TIE_REL of an E2M1
    midpoint, for given block scale codes s."""
    v, pos = _quotients(x, s, G)
    return (_near_midpoint(v, _E2M1_MIDS) & pos[:, :, None]).reshape(np.shape(x))


def quantize_fp32_order(x, G=None):
    """The same quantiser with every step an IEEE float32 operation, in this order:

      G    = fp32(amax(|x|) / 2688)            (unless a static G is given)
      enc  = 1 / (6 * G)
      s    = E4M3_rne_sat(amax_b * enc)       (0 when amax_b == 0)
      d    = dec(s) * G
      r    = 1 / d
      q_i  = E2M1_rne_sat(x_i * r)            (0 when d == 0)

    Each of 6 G, enc and amax_b * enc (and of d, r and x_i * r) rounds once, so the float32
    quotient is within 3 * 2^-24 (relative) of the exact one, and a decision can differ from
    ``quantize`` only where the exact quotient lies that close to a rounding midpoint
    (``quantize_ties`` marks every such place). Same return values as ``quantize``.
    """
    x, blocks = _blocks(x)
    rows, cols = x.shape
    G = global_scale(x) if G is None else F32(G)
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


# A quotient within this relative distance of a rounding midpoint is a tie: 8 * 2^-24,
# more than the 3 * 2^-24 that three float32 roundings (a reciprocal-multiply order) can
# move it, so any float32 evaluation order of the quotient agrees with the exact
# decision everywhere else.
TIE_REL = 2.0 ** -21

_E2M1_MIDS = (_E2M1_MAGS[:-1] + _E2M1_MAGS[1:]) / 2
_E4M3_MIDS = (_E4M3_MAGS[:-1] + _E4M3_MAGS[1:]) / 2


def _near_midpoint(v, mids, rel=TIE_REL) -> np.ndarray:
    """|v| within rel (relative) of one of the midpoints."""
    av = np.abs(np.asarray(v, np.float64))
    if len(mids) > 16:   # long tables: only the two nearest midpoints can be that close
        hi = np.clip(np.searchsorted(mids, av), 1, len(mids) - 1)
        lo = hi - 1
        return (np.abs(av - mids[lo]) <= rel * mids[lo]) | (np.abs(av - mids[hi]) <= rel * mids[hi])
    out = np.zeros(av.shape, bool)
    for m in mids:
        out |= np.abs(av - m) <= rel * m
    return out


def quantize_ties(x, G=None):
    """Where the quantisation of x is a tie (section-5 reading of the quantiser: both
    neighbouring results are correct there). Returns (block_tie (rows, cols/16),
    elem_tie (rows, cols)):

      block_tie: amax_b / (6 G) lies within TIE_REL of a midpoint between two E4M3 values,
                 so the block's scale may round either way;
      elem_tie:  x_i / d (d from the plain definition's scale) lies within TIE_REL of a
                 midpoint between two E2M1 levels.
    """
    x, blocks = _blocks(x)
    rows, cols = x.shape
    G = global_scale(x) if G is None else F32(G)
    q, s, _ = quantize(x, G)
    amax_b = np.max(np.abs(blocks), axis=2).astype(np.float64) if cols else np.zeros((rows, 0))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(amax_b > 0, amax_b / (6.0 * float(G)), 0.0)
    block_tie = _near_midpoint(np.where(np.isfinite(ratio), ratio, 0.0), _E4M3_MIDS)
    return block_tie, code_ties_for_scales(x, s, G)


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
    y = bf16(dec(q) * dec(s) * G), the dequantised value of the plain quantiser rounded
    once to bf16 (RNE; the product has at most 30 significant bits, exact in float64).
    The backward pass (straight-through estimator) is the identity and needs no oracle."""
    q, s, G = quantize(x, G)
    return bf16_round(dequantize(q, s, G)), G


def fake_quantize_fp32_order(x, G=None):
    """The float32 evaluation order of fake quantisation: codes from
    ``quantize_fp32_order``, y = bf16(fp32(fp32(e2m1(q) * e4m3(s)) * G)). The level-scale
    product is exact in float32; its product with G rounds once to float32 and then to
    bf16, which can differ from ``fake_quantize`` only at the ties ``fake_quantize_ties``
    marks."""
    q, s, G = quantize_fp32_order(x, G)
    rows, cols = q.shape
    ls = (_E2M1_TABLE[q & 0xF].reshape(rows, cols // BLOCK, BLOCK)
          * _E4M3_TABLE[np.asarray(s)][:, :, None]).reshape(rows, cols)
    y32 = ls.astype(np.float32) * np.float32(G)
    return bf16_round(y32.astype(np.float64)), G


def _near_bf16_midpoint(v, rel=2.0 ** -23) -> np.ndarray:
    """|v| within rel (relative) of a midpoint between two adjacent bf16 values (where a
    float32 intermediate rounding can decide the bf16 rounding differently)."""
    m, _ = np.frexp(np.abs(np.asarray(v, np.float64)))   # |v| = m * 2^e, 0.5 <= m < 1
    t = m * 256.0                                         # bf16 ulps: 128 <= t < 256
    return (np.abs(t - (np.floor(t) + 0.5)) <= rel * t) & (m > 0)


def fake_quantize_ties(x, G=None) -> np.ndarray:
    """Elements of fake_quantize(x, G) where both neighbouring bf16 results are correct:
    a code tie, any element of a block whose scale is a tie, or a dequantised value within
    2^-23 (relative) of a bf16 rounding midpoint."""
    bt, et = quantize_ties(x, G)
    q, s, G = quantize(x, G)
    near = _near_bf16_midpoint(dequantize(q, s, G))
    return et | np.repeat(bt, BLOCK, axis=1) | near


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
    """Quantise a bf16 GEMM operand with its own amax-derived G. Returns (codes, scales, G).

    The whole-problem functions below quantise their operands with the decisions taken in
    float32 (``quantize_fp32_order``), the precision the kernels take them in. Where that
    differs from the plain definition it is at a tie, where both results are correct, but
    a GEMM needs one fixed choice: a block scale on the other side of a tie moves all 16
    decoded values of the block by up to one scale step (12.5 %), and with the outlier
    channels such blocks shift some outputs by more than the bf16 tolerance. The
    quantiser itself is compared with the plain definition, tie rule included."""
    return quantize_fp32_order(_as_f32(x_bf16))


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
    qa, sa, _ = quantize_fp32_order(a, Ga)
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
    """Static-scale NVFP4 quantisation of bf16-valued outputs (blocks along N), the decisions
    taken in float32 like the operands of the whole-problem functions (the next GEMM's
    input)."""
    return quantize_fp32_order(np.asarray(out_bf16_values, np.float64).astype(F32), G)


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


def mx_codes_for_scales(y, e8m0) -> np.ndarray:
    """The element step of ``mx_quantize`` for given E8M0 scale codes:
    E2M1_rn_satfinite(y / 2^(e - 127)), 0 in blocks whose code is 0."""
    y = np.asarray(y, dtype=F32)
    rows, cols = y.shape
    X = e8m0_decode(e8m0)[:, :, None]
    q = e2m1_encode(y.reshape(rows, cols // MX_BLOCK, MX_BLOCK).astype(np.float64) / X)
    q = np.where((np.asarray(e8m0) > 0)[:, :, None], q, np.uint8(0)).astype(np.uint8)
    return q.reshape(rows, cols)


def mx_dequantize(codes, e8m0) -> np.ndarray:
    """dec(q) * 2^(e - 127) in float64, (rows, cols)."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    vals = _E2M1_TABLE[codes & 0xF].reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    vals *= e8m0_decode(e8m0)[:, :, None]
    return vals.reshape(rows, cols)


def _hadamard_matrix(n: int) -> np.ndarray:
    """Unnormalised Sylvester-Hadamard matrix of order n (a power of two): the Kronecker
    product H2 (x) H2 (x) ... of the 2 x 2 matrix [[1, 1], [1, -1]]."""
    h2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.kron(h2, h)
    return h


H32 = _hadamard_matrix(MX_BLOCK)


def hadamard32(x) -> np.ndarray:
    """x @ H32 per block of 32 along cols: a float64 matrix product with the Kronecker
    matrix H32 (entries +-1), rounded once to float32. H32 H32^T = 32 I, so
    (x H)(w H)^T = 32 x w^T. (The float64 sums of 32 float32 terms are exact unless a
    block's magnitudes span more than 2^24.)"""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    y = x.reshape(rows, cols // MX_BLOCK, MX_BLOCK).astype(np.float64) @ H32
    return y.reshape(rows, cols).astype(F32)


def hadamard32_fp32_order(x) -> np.ndarray:
    """The same transform as the fast Walsh-Hadamard butterfly in float32: five stages,
    stage h in (1, 2, 4, 8, 16) maps each pair (j, j + h), j with bit h clear, to
    (a + b, a - b), each sum rounded to float32. After k stages an output's error is at
    most k * 2^-24 * S, S the block's sum of |x_i|, so it lies within 6 * 2^-24 * S of
    ``hadamard32``'s result."""
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


def mx_transform_ties(x, e8m0=None):
    """Where the MXFP4 quantisation of hadamard32(x) is decided within the float32 error
    of evaluating the transform (6 * 2^-24 * S, S the block's sum of |x_i|; the band is
    8 * 2^-24 * S). Returns (block_tie (rows, cols/32), elem_tie (rows, cols)):

      block_tie: the block's amax lies within the band of a power of two (its shared
                 exponent may come out either way);
      elem_tie:  y_i / X lies within band / X of an E2M1 midpoint (X the block scale of
                 mx_quantize(hadamard32(x)), or the scales e8m0 when given).
    """
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    nb = cols // MX_BLOCK
    S = np.abs(x.reshape(rows, nb, MX_BLOCK).astype(np.float64)).sum(axis=2)
    band = 8.0 * 2.0 ** -24 * S
    y = hadamard32(x).reshape(rows, nb, MX_BLOCK).astype(np.float64)
    amax = np.abs(y).max(axis=2)
    with np.errstate(divide="ignore"):
        p = np.round(np.log2(np.where(amax > 0, amax, 1.0)))
    block_tie = (np.abs(amax - np.ldexp(1.0, p.astype(np.int64))) <= band) & (amax > 0)
    e = mx_quantize(y.reshape(rows, cols).astype(F32))[1] if e8m0 is None else np.asarray(e8m0)
    X = e8m0_decode(e)
    v = np.abs(y) / X[:, :, None]
    bx = (band / X)[:, :, None]
    elem_tie = np.zeros(v.shape, bool)
    for m in _E2M1_MIDS:
        elem_tie |= np.abs(v - m) <= bx
    return block_tie, elem_tie.reshape(rows, cols)


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
