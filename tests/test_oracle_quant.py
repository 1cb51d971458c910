"""Pins for the oracle's NVFP4 block quantiser and storage layouts (CPU only)."""
import numpy as np
import pytest

from oracle import nvfp4_oracle as o
import workloads as wk


def _rand(rows, cols, seed=0, outliers=0):
    return wk.activations(rows, cols, outliers, seed).float().numpy()


def test_global_scale_puts_largest_block_scale_on_448():
    x = _rand(64, 256, outliers=2)
    q, s, G = o.quantize(x)
    assert G == np.float32(np.max(np.abs(x)) / np.float32(2688))
    assert s.max() == 0x7E                       # 448
    # the block holding the tensor's amax uses the top scale
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert s[r, c // 16] == 0x7E
    # and its amax element maps to the top level (magnitude code 7, value 6)
    assert q[r, c] & 7 == 7


def test_idempotent_on_dequantised_values():
    x = _rand(128, 512, seed=3, outliers=4)
    q, s, G = o.quantize(x)
    deq = o.dequantize(q, s, G).astype(np.float32)
    q2, s2, G2 = o.quantize(deq, G)
    assert np.array_equal(q2 & 7, q & 7)          # magnitudes
    nz = (q & 7) != 0
    assert np.array_equal(q2[nz], q[nz])          # signs where nonzero
    assert np.array_equal(s2, s)


def test_per_element_error_is_within_half_a_level_step():
    x = _rand(64, 1024, seed=5, outliers=3)
    q, s, G = o.quantize(x)
    d = (o.e4m3_decode(s).astype(np.float32) * G).astype(np.float64)
    dd = np.repeat(d, 16, axis=1)
    t = np.abs(x.astype(np.float64)) / dd          # magnitude in level units
    half = np.where(t < 2, 0.25, np.where(t < 4, 0.5, 1.0))
    err = np.abs(np.abs(o.e2m1_decode(q)) - t)
    sat = t > 6
    assert np.all(err[~sat] <= half[~sat] * (1 + 1e-6))
    assert np.all(q[sat] & 7 == 7)


def test_zero_blocks_and_zero_tensor():
    x = _rand(4, 64, seed=1)
    x[1, 16:32] = 0
    q, s, G = o.quantize(x)
    assert s[1, 1] == 0 and np.all(q[1, 16:32] == 0)
    q0, s0, G0 = o.quantize(np.zeros((4, 64), np.float32))
    assert G0 == 0 and not q0.any() and not s0.any()


def test_static_scale_saturates_instead_of_overflowing():
    x = _rand(4, 64, seed=2)
    G = np.float32(np.max(np.abs(x)) / 2688 / 8)   # 8x too small
    q, s, _ = o.quantize(x, G)
    assert s.max() == 0x7E
    assert np.all(np.isfinite(o.dequantize(q, s, G)))


def test_row_permutation_commutes_with_quantisation():
    w = wk.weights(64, 256, 0.05, seed=4).float().numpy()
    q, s, G = o.quantize(w)
    qi, si, Gi = o.quantize(o.interleave_gate_up(w))
    assert G == Gi
    assert np.array_equal(qi, o.interleave_gate_up(q))
    assert np.array_equal(si, o.interleave_gate_up(s))


def test_dequantised_error_is_fp4_sized():
    x = _rand(256, 1024, seed=6)
    q, s, G = o.quantize(x)
    deq = o.dequantize(q, s, G)
    rel = np.linalg.norm(deq - x) / np.linalg.norm(x)
    assert 0.05 < rel < 0.15


def test_interleave_is_a_bijection_pairing_gate_and_up():
    nh = 8
    rows = np.arange(2 * nh)
    p = o.interleave_gate_up(rows)
    assert sorted(p.tolist()) == rows.tolist()
    assert np.array_equal(p[0::2], np.arange(nh))
    assert np.array_equal(p[1::2], np.arange(nh) + nh)


@pytest.mark.parametrize("rows,cols", [(128, 64), (256, 512), (130, 80), (1, 16)])
def test_scale_layout_is_a_bijection_onto_the_buffer(rows, cols):
    nkb = cols // 16
    rp = ((rows + 127) // 128) * 128
    kp = ((nkb + 3) // 4) * 4
    rr, kk = np.meshgrid(np.arange(rp), np.arange(kp), indexing="ij")
    off = o.sf_offset(rr, kk, cols)
    assert off.min() == 0 and off.max() == o.sf_bytes(rows, cols) - 1
    assert len(np.unique(off)) == off.size
    # every 128-row x 4-block unit is one contiguous 512-byte range
    for r0 in range(0, rp, 128):
        for k0 in range(0, kp, 4):
            u = off[r0:r0 + 128, k0:k0 + 4]
            assert u.max() - u.min() == 511 and u.min() % 512 == 0
    # within a unit, 32 consecutive rows are 16 bytes apart (one line each)
    assert np.all(np.diff(off[:32, 0]) == 16)


def test_scale_and_code_packing_roundtrip():
    rng = np.random.default_rng(0)
    s = rng.integers(0, 0x7F, size=(200, 12), dtype=np.uint8)
    buf = o.pack_scales(s, 192)
    assert np.array_equal(o.unpack_scales(buf, 200, 192), s)
    c = rng.integers(0, 16, size=(5, 64), dtype=np.uint8)
    p = o.pack_codes(c)
    assert p.shape == (5, 32)
    assert np.array_equal(p[:, 0] & 0xF, c[:, 0]) and np.array_equal(p[:, 0] >> 4, c[:, 1])
    assert np.array_equal(o.unpack_codes(p), c)


# ---- fake quantisation (quantise-dequantise) -------------------------------------

def _representable(rows, cols, G, seed):
    """Blocks whose largest magnitude is 6 * e4m3(s) * G: every element is level * scale * G,
    exactly, for a power-of-two G."""
    rng = np.random.default_rng(seed)
    lv = o.e2m1_decode(np.arange(16))
    q = rng.integers(0, 16, size=(rows, cols))
    q[:, ::16] = 7  # the block maximum (+6)
    s = rng.integers(0x20, 0x7E, size=(rows, cols // 16))  # normal E4M3 scales
    x = lv[q] * np.repeat(o.e4m3_decode(s), 16, axis=1) * float(G)
    return x.astype(np.float32)


def test_fake_quantize_returns_representable_values_unchanged():
    G = np.float32(2.0 ** -7)
    x = _representable(64, 256, G, seed=1)
    y, G2 = o.fake_quantize(x, G)
    assert G2 == G
    # level * scale * G has at most 7 significant bits here, so bf16 holds it exactly
    assert np.array_equal(y, x.astype(np.float64))


def test_fake_quantize_is_idempotent_at_power_of_two_scale():
    G = np.float32(2.0 ** -9)
    x = _rand(128, 512, seed=8, outliers=2)
    y, _ = o.fake_quantize(x, G)
    y2, _ = o.fake_quantize(y.astype(np.float32), G)
    assert np.array_equal(y2, y)


def test_fake_quantize_is_odd_and_close_to_the_exact_dequantisation():
    x = _rand(64, 512, seed=9, outliers=3)
    y, G = o.fake_quantize(x)
    yn, Gn = o.fake_quantize(-x)
    assert Gn == G and np.array_equal(yn, -y)
    q, s, _ = o.quantize(x)
    exact = o.dequantize(q, s, G)  # float64, no rounding
    # one fp32 and one bf16 rounding: within 2^-8 relative (plus fp32 underflow slack)
    assert np.all(np.abs(y - exact) <= 2.0 ** -8 * np.abs(exact) + 1e-30)
    # and the fake-quantised tensor stays within half a level step of x (FP4-sized error)
    assert np.abs(y - x).max() <= 0.5 * 2.0 * 448 * float(G) * 1.01


def test_fake_quantize_of_zero_is_zero():
    y, G = o.fake_quantize(np.zeros((128, 64), np.float32))
    assert G == 0 and not y.any()


# ---- MXFP4 and the block Hadamard transform ---------------------------------------

def test_hadamard32_matches_scipy_and_is_its_own_inverse_up_to_32():
    import scipy.linalg
    H = scipy.linalg.hadamard(32).astype(np.float64)  # Sylvester construction, a library routine
    x = _rand(16, 128, seed=12)
    y = o.hadamard32(x)
    ref = (x.astype(np.float64).reshape(16, 4, 32) @ H).reshape(16, 128)
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-5)
    xi = np.random.default_rng(2).integers(-8, 8, size=(8, 64)).astype(np.float32)  # exact in fp32
    assert np.array_equal(o.hadamard32(o.hadamard32(xi)), 32 * xi)
    assert np.array_equal((xi.reshape(8, 2, 32).astype(np.float64) @ H).reshape(8, 64), o.hadamard32(xi))


def test_mx_quantize_scale_rule_and_bounds():
    x = _rand(64, 256, seed=13, outliers=2)
    q, e = o.mx_quantize(x)
    xb = x.reshape(64, 8, 32)
    amax = np.abs(xb).max(axis=2)
    X = o.e8m0_decode(e)
    # the shared exponent puts amax / X in [4, 8): one power of two below E2M1's top level
    assert np.all((amax / X >= 4) & (amax / X < 8))
    deq = o.mx_dequantize(q, e)
    # error within half the widest level step (2) of the block, or the saturation of
    # values above 6 X
    err = np.abs(deq - x).reshape(64, 8, 32)
    bound = np.maximum(1.0 * X, amax - 6 * X)[:, :, None]
    assert np.all(err <= bound + 1e-12)
    # exact on representable blocks: levels times a power of two, top level present
    lv = o.e2m1_decode(np.arange(16))
    qq = np.random.default_rng(1).integers(0, 16, size=(4, 64))
    qq[:, ::32] = 7
    xr = (lv[qq] * 2.0 ** -5).astype(np.float32)
    q2, e2 = o.mx_quantize(xr)
    assert np.array_equal(o.mx_dequantize(q2, e2), xr.astype(np.float64))
    assert np.all(e2 == 127 - 5)


def test_mx_zero_block_and_layout_roundtrip():
    x = _rand(128, 256, seed=14)
    x[3, 32:64] = 0
    q, e = o.mx_quantize(x)
    assert e[3, 1] == 0 and not q[3, 32:64].any()
    buf = o.mx_pack_scales(e, 256)
    assert buf.size == o.mx_sf_bytes(128, 256) == 128 * 8
    assert np.array_equal(o.mx_unpack_scales(buf, 128, 256), e)


# ---- the plain definition against exact rational arithmetic, and the float32 order ----

from fractions import Fraction  # noqa: E402

_E4M3_VALUES = [(Fraction(float(v)), c) for c, v in enumerate(o.e4m3_decode(np.arange(0x7F)))]
_E2M1_VALUES = [(Fraction(float(v)), c) for c, v in enumerate(o.e2m1_decode(np.arange(8)))]


def _nearest_code(value, table):
    """Brute force: the table entry nearest to an exact rational, ties to the even code
    (the even mantissa). Anything past the last entry lands on it (saturation)."""
    best = min(abs(value - t) for t, _ in table)
    cands = [c for t, c in table if abs(value - t) == best]
    return min(cands, key=lambda c: (c % 2, c))


def _quantize_rational(x, G):
    """NVFP4 quantisation in exact rational arithmetic, one element at a time."""
    rows, cols = x.shape
    Gf = Fraction(float(G))
    q = np.zeros((rows, cols), np.uint8)
    s = np.zeros((rows, cols // 16), np.uint8)
    for r in range(rows):
        for b in range(cols // 16):
            blk = x[r, 16 * b:16 * b + 16]
            amax = max(abs(Fraction(float(v))) for v in blk)
            if amax == 0:
                sc = 0
            elif Gf == 0:
                sc = 0x7E
            else:
                sc = _nearest_code(amax / (6 * Gf), _E4M3_VALUES)
            s[r, b] = sc
            d = Fraction(float(o.e4m3_decode(sc))) * Gf
            for i, v in enumerate(blk):
                if d == 0:
                    continue
                code = _nearest_code(abs(Fraction(float(v))) / d, _E2M1_VALUES)
                q[r, 16 * b + i] = code | (8 if np.signbit(v) else 0)
    return q, s


def _near_tie_blocks(rows, seed):
    """Blocks built around rounding midpoints: element 0 fixes the block scale at a chosen
    E4M3 code, the other 15 sit within 3 float32 ulps of (E2M1 midpoint) * d."""
    rng = np.random.default_rng(seed)
    G = np.float32(rng.uniform(1e-3, 1e-2))
    s_code = rng.integers(0x20, 0x70, size=rows)
    d = o.e4m3_decode(s_code) * float(G)
    x = np.zeros((rows, 16), np.float32)
    x[:, 0] = (6 * d).astype(np.float32)
    mids = (o.e2m1_decode(np.arange(7)) + o.e2m1_decode(np.arange(1, 8))) / 2
    base = (mids[rng.integers(0, 7, size=(rows, 15))] * d[:, None]).astype(np.float32)
    steps = rng.integers(-3, 4, size=(rows, 15))
    bits = base.view(np.int32) + steps.astype(np.int32)     # +-k ulps (all positive values)
    x[:, 1:] = bits.view(np.float32)
    x[:, 1::2] *= -1
    return x, G


def _near_scale_tie_blocks(rows, seed):
    """Blocks whose amax / (6 G) lies within 3 float32 ulps of a midpoint between two E4M3
    scales (normal and subnormal), the other elements spread below the amax."""
    rng = np.random.default_rng(seed)
    G = np.float32(rng.uniform(1e-3, 1e-2))
    lo = rng.integers(0x01, 0x7D, size=rows)
    mid4 = (o.e4m3_decode(lo) + o.e4m3_decode(lo + 1)) / 2
    amax = (6 * mid4 * float(G)).astype(np.float32)
    amax = (amax.view(np.int32) + rng.integers(-3, 4, size=rows).astype(np.int32)).view(np.float32)
    x = (rng.uniform(-1, 1, size=(rows, 16)) * amax[:, None]).astype(np.float32)
    x[:, 0] = amax
    return x, G


def _exact_ties():
    """Exact midpoints at a power-of-two G: every quotient is exact in binary, so both
    neighbours are equally near and the even code must win."""
    G = np.float32(2.0 ** -6)
    mids2 = (o.e2m1_decode(np.arange(7)) + o.e2m1_decode(np.arange(1, 8))) / 2
    x = np.zeros((4, 32), np.float32)
    x[0, 0] = 6 * float(G)                       # scale 1.0 (code 0x38)
    x[0, 1:8] = mids2 * float(G)
    x[0, 8:15] = -mids2 * float(G)
    mids4 = (o.e4m3_decode(np.array([0x38, 0x39, 0x3A])) + o.e4m3_decode(np.array([0x39, 0x3A, 0x3B]))) / 2
    x[1, 0] = 6 * mids4[0] * float(G)            # amax / (6 G) exactly between two scales
    x[1, 16] = 6 * mids4[1] * float(G)
    x[2, 0] = 6 * mids4[2] * float(G)
    x[2, 16] = 6 * 2.0 ** -10 * float(G)         # between scale 0 and the smallest subnormal
    x[3, 0] = 6 * 3 * 2.0 ** -10 * float(G)      # subnormal scales
    x[3, 1:4] = [1e-7, -2e-7, 3e-7]
    return x, G


def test_quantize_is_the_exact_rational_rounding():
    """The plain quantiser equals nearest-value rounding done in exact rational arithmetic
    on: workload-distributed blocks with a dynamic scale, blocks built within 3 ulps of
    every E2M1 midpoint, exact midpoints of codes and of scales (including the subnormal
    scales), a saturating static scale and zero blocks."""
    cases = []
    x = _rand(6, 64, seed=31, outliers=2)
    cases.append((x, o.global_scale(x)))
    cases.append(_near_tie_blocks(48, seed=32))
    cases.append(_near_scale_tie_blocks(48, seed=34))
    cases.append(_exact_ties())
    xs = _rand(4, 64, seed=33)
    xs[1, 16:32] = 0
    cases.append((xs, np.float32(o.global_scale(xs) / 16)))   # saturates
    cases.append((xs, np.float32(0.0)))                        # no scale: codes all zero
    for x, G in cases:
        q, s, _ = o.quantize(x, G)
        qr, sr = _quantize_rational(x, G)
        assert np.array_equal(s, sr)
        assert np.array_equal(q, qr)


def test_exact_ties_take_the_even_code():
    x, G = _exact_ties()
    q, s, _ = o.quantize(x, G)
    assert s[0, 0] == 0x38
    # midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 -> levels 0, 1, 1, 2, 2, 4, 4
    assert q[0, 1:8].tolist() == [0, 2, 2, 4, 4, 6, 6]
    assert q[0, 8:15].tolist() == [8 | c for c in (0, 2, 2, 4, 4, 6, 6)]
    assert s[1, 0] == 0x38 and s[1, 1] == 0x3A and s[2, 0] == 0x3A
    assert s[2, 1] == 0x00                     # 2^-10 lies halfway between 0 and 2^-9
    assert s[3, 0] == 0x02                     # 3 * 2^-10 between 2^-9 and 2^-8: even code


def test_fp32_order_differs_from_the_plain_definition_only_at_ties():
    """The float32 reciprocal-multiply order against the plain definition: on blocks built
    next to midpoints the two orders disagree (so the tie rule matters), and everywhere,
    on those blocks and on workload activations and weights, a disagreement lies inside
    quantize_ties' band and moves a code by one level."""
    cases = [_near_tie_blocks(2048, seed=41), _near_scale_tie_blocks(2048, seed=45),
             (_rand(512, 3072, seed=42, outliers=3), None),
             (wk.weights(1024, 3072, 1 / np.sqrt(3072), seed=43).float().numpy(), None)]
    diffs, sdiffs = [], []
    for x, G in cases:
        q, s, Gp = o.quantize(x, G)
        q2, s2, G2 = o.quantize_fp32_order(x, G)
        bt, et = o.quantize_ties(x, G)
        assert Gp == G2
        assert not ((s != s2) & ~bt).any()
        assert np.all(np.abs(s.astype(int) - s2.astype(int)) <= 1)
        sdiffs.append(int((s != s2).sum()))
        same_scale = np.repeat(s == s2, 16, axis=1)
        dq = (q != q2) & same_scale
        assert not (dq & ~et).any()
        lvl = lambda c: np.where(c & 8, -1, 1) * (c & 7).astype(np.int64)
        assert np.all(np.abs(lvl(q) - lvl(q2))[dq] <= 1)
        diffs.append(int(dq.sum()))
    assert diffs[0] > 0 and sdiffs[1] > 0


def test_ties_band_is_tight_enough_to_matter():
    """The band exempts a small share of workload elements, not everything. (Ties are not
    rare: G = amax / (6 * 448) makes x / d a ratio of short bf16 numbers, which often sits
    on a midpoint except for the float32 rounding of G.)"""
    x = _rand(256, 3072, seed=44, outliers=3)
    bt, et = o.quantize_ties(x)
    assert et.mean() < 1e-2 and bt.mean() < 1e-3


def test_fake_quantize_fp32_order_differs_only_at_ties():
    for x, G in [_near_tie_blocks(1024, seed=51), (_rand(256, 1024, seed=52, outliers=2), None)]:
        y, _ = o.fake_quantize(x, G)
        y2, _ = o.fake_quantize_fp32_order(x, G)
        t = o.fake_quantize_ties(x, G)
        assert not ((y != y2) & ~t).any()


def test_hadamard_matrix_is_the_library_one_and_orthogonal():
    import scipy.linalg
    H = scipy.linalg.hadamard(32).astype(np.float64)   # a library routine
    assert np.array_equal(o.H32, H)
    assert np.array_equal(o.H32 @ o.H32.T, 32 * np.eye(32))
    # the transform of a unit vector is the matching row of H
    e = np.zeros((32, 32), np.float32)
    e[np.arange(32), np.arange(32)] = 1
    assert np.array_equal(o.hadamard32(e), H.astype(np.float32))


def _wide_blocks(rows, seed):
    """Blocks mixing magnitudes 2^0 .. 2^-22 with 8-bit mantissas: partial sums of 32 such
    terms need more than float32's 24 bits, so a butterfly in float32 rounds on the way."""
    rng = np.random.default_rng(seed)
    m = rng.integers(128, 256, size=(rows, 64)) / 128.0
    e = rng.integers(-22, 1, size=(rows, 64))
    sign = rng.choice([-1.0, 1.0], size=(rows, 64))
    return (sign * np.ldexp(m, e)).astype(np.float32)


def test_hadamard32_is_the_exact_sum_rounded_once():
    x = np.concatenate([_rand(4, 64, seed=61, outliers=1), _wide_blocks(4, seed=63)])
    y = o.hadamard32(x)
    assert not np.array_equal(y, o.hadamard32_fp32_order(x))   # the butterfly rounds here
    for r in range(8):
        for b in range(2):
            for j in range(32):
                exact = sum(Fraction(float(x[r, 32 * b + i])) * int(o.H32[i, j]) for i in range(32))
                assert Fraction(float(exact)) == exact          # fits a float64 exactly
                assert y[r, 32 * b + j] == np.float32(float(exact))


def test_hadamard_butterfly_and_mx_codes_differ_only_within_the_float32_bound():
    x = _rand(512, 1024, seed=62, outliers=2)
    y = o.hadamard32(x).astype(np.float64)
    yb = o.hadamard32_fp32_order(x).astype(np.float64)
    S = np.repeat(np.abs(x.reshape(512, 32, 32).astype(np.float64)).sum(axis=2), 32, axis=1)
    assert np.all(np.abs(y - yb) <= 6 * 2.0 ** -24 * S)
    q, e = o.mx_quantize(y.astype(np.float32))
    qb, eb = o.mx_quantize(yb.astype(np.float32))
    bt, et = o.mx_transform_ties(x)
    assert not ((e != eb) & ~bt).any()
    same = np.repeat(e == eb, 32, axis=1)
    assert not ((q != qb) & same & ~et).any()
