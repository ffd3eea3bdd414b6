"""The GPU tests' near-tie rule for the intermediate's E4M3 codes
(tests/parity.py), exercised on the CPU with planted code changes."""
import numpy as np
import pytest

from oracle import moe as O
from tests.parity import near_tie_rows


def _case():
    rng = np.random.default_rng(5)
    a32 = np.float32(rng.standard_normal((4, 256))).astype(np.float64)
    # a value whose x = a / scale sits on the boundary between 1.0 and 1.125
    hq, hs = O.quant_1x128(a32)
    a32[2, 7] = 1.0625 * hs[2, 0] * (1 + 1e-7)
    a32[3, 9] = 1.03 * hs[3, 0]                  # far from every boundary
    hq, hs = O.quant_1x128(a32)
    return a32, hq, hs


def test_identical_intermediate_has_no_near_ties():
    a32, hq, hs = _case()
    rows, dist = near_tie_rows(hq.copy(), hs.copy(), a32, hq, hs, "same")
    assert rows.size == 0 and dist == 0.0


def test_adjacent_code_at_a_boundary_is_accepted():
    a32, hq, hs = _case()
    g = hq.copy()
    assert g[2, 7] == 0x39                       # 1.125 (ties to the even mantissa)
    g[2, 7] = 0x38                               # 1.0: the other side of the tie
    rows, dist = near_tie_rows(g, hs, a32, hq, hs, "near tie")
    assert list(rows) == [2] and dist < 1e-6


def test_code_change_away_from_a_boundary_is_rejected():
    a32, hq, hs = _case()
    g = hq.copy()
    g[3, 9] += 1
    with pytest.raises(AssertionError, match="away from a rounding boundary"):
        near_tie_rows(g, hs, a32, hq, hs, "far")


def test_code_two_steps_away_is_rejected():
    a32, hq, hs = _case()
    g = hq.copy()
    g[2, 7] -= 2
    with pytest.raises(AssertionError, match="more than one step"):
        near_tie_rows(g, hs, a32, hq, hs, "two steps")


def test_scale_mismatch_is_rejected():
    a32, hq, hs = _case()
    s = hs.copy()
    s[1, 1] *= 1.001
    with pytest.raises(AssertionError, match="scale"):
        near_tie_rows(hq, s, a32, hq, hs, "scale")
