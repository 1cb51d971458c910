"""CPU checks of the GPU tests' comparison helpers (tests/gpu_util.py): the tie rule accepts
what the float32 evaluation order produces and rejects a planted mistake outside a tie, so
the GPU parity tests cannot pass a wrong kernel for the helpers' sake."""
import numpy as np
import pytest

from oracle import nvfp4_oracle as o
import workloads as wk
from gpu_util import assert_close_chain, assert_nvfp4_plain, assert_requant_point13, level_index


def _weights():
    # seed 3: the float32 order and the plain definition disagree on ~1 % of the scales
    return wk.weights(512, 3072, 1 / np.sqrt(3072), seed=3).float().numpy()


def test_level_index_is_signed_and_merges_the_zeros():
    assert level_index(np.array([0, 8, 1, 9, 7, 15])).tolist() == [0, 0, 1, -1, 7, -7]


def test_plain_rule_accepts_the_float32_order():
    x = _weights()
    q, s, G = o.quantize_fp32_order(x)
    scales, codes = assert_nvfp4_plain(q, s, x, G, "fp32 order")
    assert scales + codes > 0          # the tie exemptions are really used here


def test_plain_rule_rejects_a_code_off_a_tie():
    x = _weights()
    q, s, G = o.quantize_fp32_order(x)
    bt, et = o.quantize_ties(x, G)
    q_ref, s_ref, _ = o.quantize(x, G)
    ok = (~et) & np.repeat(~bt & (s == s_ref), 16, axis=1) & ((q & 7) > 0) & ((q & 7) < 7)
    r, c = np.argwhere(ok)[0]
    bad = q.copy()
    bad[r, c] = (bad[r, c] & 8) | ((bad[r, c] & 7) + 1)   # one level up, not at a tie
    with pytest.raises(AssertionError):
        assert_nvfp4_plain(bad, s, x, G, "planted code")


def test_plain_rule_rejects_a_scale_off_a_tie():
    x = _weights()
    q, s, G = o.quantize_fp32_order(x)
    bt, _ = o.quantize_ties(x, G)
    r, b = np.argwhere(~bt & (s > 0x10) & (s < 0x70))[0]
    bad = s.copy()
    bad[r, b] += 1
    with pytest.raises(AssertionError):
        assert_nvfp4_plain(q, bad, x, G, "planted scale")


def test_requant_rule_accepts_equal_bf16_and_rejects_two_levels():
    y = o.bf16_round(wk.activations(256, 1024, 0, seed=4).float().numpy().astype(np.float64) * 0.3)
    G = np.float32(np.abs(y).max() / 2688)
    q, s, _ = o.quantize_fp32_order(y.astype(np.float32), G)
    assert assert_requant_point13(q, s, y, y, G, "same bf16") == 0.0
    bad = q.copy()
    r, c = np.argwhere(((q & 7) > 1) & ((q & 7) < 6))[0]
    bad[r, c] = (bad[r, c] & 8) | ((bad[r, c] & 7) - 2)
    with pytest.raises(AssertionError):
        assert_requant_point13(bad, s, y, y, G, "planted")


def test_chain_rule_bounds():
    ref = np.random.default_rng(0).standard_normal((64, 256))
    rms = np.sqrt(np.mean(ref * ref))
    assert_close_chain(ref + 0.5e-3 * rms, ref, "within both bounds")
    with pytest.raises(AssertionError):   # every element inside its own bound, not the norm
        assert_close_chain(ref + 1.5e-2 * rms, ref, "normwise over")
    with pytest.raises(AssertionError):
        assert_close_chain(ref + np.where(np.arange(256) == 7, 0.05 * rms, 0.0), ref, "one element over")
