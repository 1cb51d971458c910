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
