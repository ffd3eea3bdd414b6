"""Pins for the oracle's number formats (E4M3, bf16, fp32), CPU only.

The E4M3 encoder is checked against (a) the format's published values
(tests/golden/e4m3_spec_values.txt), (b) an exhaustive nearest-value search
with the ties-to-even rule, written here from the definition, and (c) torch's
own float8_e4m3fn cast, an independent library routine.
"""
import os

import numpy as np
import pytest
import torch

from oracle.e4m3 import (E4M3_MAX, decode, decode_table, encode, round_bf16,
                         round_fp32)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _spec_rows():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_spec_values.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            code, _bits, val = line.split()
            rows.append((int(code, 16), float(val)))
    return rows


def test_decode_matches_published_values():
    rows = _spec_rows()
    assert len(rows) == 10
    for code, val in rows:
        got = decode(np.array([code]))[0]
        if np.isnan(val):
            assert np.isnan(got)
        else:
            assert got == val
            assert np.signbit(got) == np.signbit(val)


def test_positive_codes_are_monotone_and_max_is_448():
    t = decode_table()
    pos = t[:127]
    assert np.all(np.diff(pos) > 0)
    assert pos[-1] == E4M3_MAX == 448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    # negative half mirrors the positive half
    assert np.array_equal(t[128:255], -t[:127])


def test_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(encode(decode(codes)), codes)


def _brute_force_encode(x):
    """Nearest finite E4M3 value by exhaustive search; ties -> even code;
    magnitudes above 448 saturate."""
    t = decode_table()
    finite = [c for c in range(127)]          # positive codes 0..126
    out = np.empty(len(x), np.uint8)
    for i, v in enumerate(x):
        a = min(abs(v), 448.0)
        best, bd = None, None
        for c in finite:
            dd = abs(t[c] - a)
            if bd is None or dd < bd or (dd == bd and c % 2 == 0):
                best, bd = c, dd
        out[i] = best | (0x80 if np.signbit(v) else 0)
    return out


def _hard_cases():
    t = decode_table()[:127]
    mids = (t[:-1] + t[1:]) / 2.0             # exact ties
    cases = [mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), t,
             np.array([0.0, -0.0, 448.0, 449.0, 463.9, 464.0, 465.0, 1e6,
                       2.0 ** -10, 2.0 ** -9 * 0.5, 2.0 ** -9 * 0.5000001])]
    x = np.concatenate(cases)
    x = np.concatenate([x, -x])
    return round_fp32(x)


def test_encode_matches_exhaustive_search_on_ties_and_edges():
    x = _hard_cases()
    assert np.array_equal(encode(x), _brute_force_encode(x))


def test_encode_matches_exhaustive_search_random():
    rng = np.random.default_rng(1)
    x = round_fp32(np.concatenate([
        rng.uniform(-500, 500, 3000),
        np.exp2(rng.uniform(-12, 9, 3000)) * rng.choice([-1, 1], 3000)]))
    assert np.array_equal(encode(x), _brute_force_encode(x))


def test_encode_matches_torch_float8_cast():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        _hard_cases(),
        np.exp2(rng.uniform(-14, 8.8, 200000)) * rng.choice([-1, 1], 200000),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448.0]        # torch's cast does not saturate
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(encode(x.astype(np.float64)), ref)


def test_encode_saturates():
    got = encode(np.array([448.0, 460.0, 464.0, 1e9, -1e9, -500.0]))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(100000) * 10.0,
        np.exp2(rng.uniform(-140, 100, 50000)) * rng.choice([-1, 1], 50000),
    ]).astype(np.float32)
    # exact bf16 ties: bf16 value + half a bf16 ulp
    b = torch.from_numpy(rng.standard_normal(1000).astype(np.float32)).to(torch.bfloat16)
    bb = b.to(torch.float32).numpy()
    ulp = np.abs(bb) * 2.0 ** -8
    ties = (bb + np.sign(bb) * ulp * 0.5).astype(np.float32)
    x = np.concatenate([x, ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(round_bf16(x.astype(np.float64)), ref)


def test_round_fp32_is_nearest():
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 1.0 + 2.0 ** -30])
    assert list(round_fp32(x)) == [1.0, 1.0 + 2.0 ** -22, 1.0]


@pytest.mark.parametrize("v,code", [(1.0, 0x38), (-2.0, 0xC0), (0.5, 0x30),
                                    (2.0 ** -7, 0x04), (240.0, 0x77)])
def test_encode_known_values(v, code):
    assert encode(np.array([v]))[0] == code
