"""The GPU tests' near-tie rule for the intermediate's E4M3 codes
(tests/parity.py), exercised on the CPU with planted code changes."""
import numpy as np
import pytest

from oracle import moe as O
from tests.parity import accumulation_bound, near_tie_rows


def _case():
    rng = np.random.default_rng(5)
    a32 = np.float32(rng.standard_normal((4, 256))).astype(np.float64)
    hq, hs = O.quant_1x128(a32)
    # x = a / scale just above the boundary between 1.0 and 1.125, and one
    # far from every boundary
    a32[2, 7] = 1.0625 * hs[2, 0] * (1 + 1e-7)
    a32[3, 9] = 1.03 * hs[3, 0]
    hq, hs = O.quant_1x128(a32)
    da = np.abs(a32) * 1e-6                    # a bound of one part in a million
    return a32, da, hq, hs


def test_identical_intermediate_has_no_near_ties():
    a32, da, hq, hs = _case()
    rows, dist = near_tie_rows(hq.copy(), hs.copy(), a32, da, hq, hs, "same")
    assert rows.size == 0 and dist == 0.0


def test_other_side_of_a_boundary_within_the_bound_is_accepted():
    a32, da, hq, hs = _case()
    g = hq.copy()
    assert g[2, 7] == 0x39                       # 1.125
    g[2, 7] = 0x38                               # 1.0: the other side of the boundary
    rows, dist = near_tie_rows(g, hs, a32, da, hq, hs, "near tie")
    assert list(rows) == [2] and dist < 1.0


def test_code_change_beyond_the_bound_is_rejected():
    a32, da, hq, hs = _case()
    for r, c, step in [(3, 9, 1), (2, 7, -2)]:
        g = hq.copy()
        g[r, c] = np.uint8(int(g[r, c]) + step)
        with pytest.raises(AssertionError, match="outside the accumulation bound"):
            near_tie_rows(g, hs, a32, da, hq, hs, "far")


def test_scale_mismatch_is_rejected():
    a32, da, hq, hs = _case()
    s = hs.copy()
    s[1, 1] *= 1.001
    with pytest.raises(AssertionError, match="scale"):
        near_tie_rows(hq, s, a32, da, hq, hs, "scale")


def test_accumulation_bound_grows_with_the_absolute_sums():
    # one expert, two rows: the bound is proportional to sum |x w| and
    # vanishes where U = 0 and silu(G) = 0
    d = I = 128
    xq = np.full((2, d), 0x38, np.uint8)
    xs = np.array([[1.0], [2.0]])
    w = dict(gate_q=np.full((I, d), 0x04, np.uint8), gate_s=np.ones((1, 1)),
             up_q=np.full((I, d), 0x04, np.uint8), up_s=np.ones((1, 1)),
             down_q=np.full((d, I), 0x04, np.uint8), down_s=np.ones((1, 1)))
    p = O.expert_ffn_parts(xq, xs, w)
    da = accumulation_bound(xq, xs, w, p["G"], p["U"])
    assert np.all(da > 0) and np.all(da[1] > 2 * da[0])
    zero = accumulation_bound(xq, xs, w, np.zeros((2, I)), np.zeros((2, I)))
    assert np.all(zero == 0.0)


def test_bf16_output_rule():
    from oracle.e4m3 import round_bf16
    from tests.parity import assert_bf16_rounding
    rng = np.random.default_rng(3)
    ref = rng.standard_normal(1000)
    # the correctly rounded outputs pass with any bound, and count no flips
    assert assert_bf16_rounding(round_bf16(ref), ref, 0.0, "exact") == 0
    # one bf16 step off is rejected when the bound is far below a step
    step = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)
    with pytest.raises(AssertionError):
        assert_bf16_rounding(round_bf16(ref) + step, ref, 1e-12, "one step off")
    # a value just above a bf16 midpoint may come out on either side when the
    # bound reaches the midpoint, and not when it does not
    mid = 1.0 + 2.0 ** -8                       # between 1 and 1 + 2^-7
    v = np.array([mid + 2.0 ** -30])
    assert assert_bf16_rounding(np.array([1.0]), v, 2.0 ** -29, "near tie") == 1
    with pytest.raises(AssertionError):
        assert_bf16_rounding(np.array([1.0]), v, 2.0 ** -31, "outside the bound")


def test_bf16_output_rule_rejects_truncation():
    # a kernel that truncated its FP32 sums to bf16 instead of rounding to
    # nearest even is caught, even with a generous accumulation bound
    from tests.parity import assert_bf16_rounding
    rng = np.random.default_rng(4)
    ref = rng.standard_normal(4096)
    bits = ref.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    truncated = bits.view(np.float32).astype(np.float64)
    with pytest.raises(AssertionError):
        assert_bf16_rounding(truncated, ref, 1e-9 * np.abs(ref), "truncated")
