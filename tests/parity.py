"""Parity helpers shared by the GPU tests.

Tolerance for floating-point outputs: |gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref).

Requantisation near-ties. The expert intermediate a = silu(G) * U is
accumulated by the kernel in FP32 (each 128-wide K block promoted in FP32) and
by the oracle in float64, so the two differ by FP32 rounding. Its E4M3 code
(1x128 tiles along I) is an integer decided by floating point, so where the
kernel's value may lie on the other side of a rounding boundary, both codes
are valid outcomes of the method. The rule, per element: from the oracle's G,
U and the sums of absolute products behind them, bound how far the kernel's
FP32 value of x = a / scale can be from the oracle's (accumulation_bound);
the kernel's code must be one that some value within that distance rounds
to. All other codes must equal the oracle's, the tile scales must agree to
SCALE_RTOL, and a row holding an accepted different code is re-evaluated by
the oracle's down projection on the kernel's codes (as a token whose top-K
keys tie within the routing margin is evaluated under the kernel's
selection) before its output is compared.

bf16 expert outputs. The kernel sums each output in FP32 and rounds it to
bf16 (nearest even); the oracle's value is float64. From the sum of absolute
products behind it (down_bound), the kernel's FP32 value lies within a bound
of the oracle's, so its bf16 output must lie between the bf16 roundings of
the two ends of that interval (assert_bf16_rounding): equal to the oracle's
rounding except where the oracle's value sits within the bound of a bf16
midpoint, where either neighbour is valid. h' is then compared with the
oracle's combine of the kernel's (so validated) bf16 outputs.
"""
import numpy as np

from oracle import moe as O
from oracle.e4m3 import decode, encode, round_bf16

RTOL, ATOL_RMS = 8e-3, 1e-3
SCALE_RTOL = 1e-4        # tile scales fl32(amax / 448): amax accumulated in FP32 vs float64
EPS32 = 2.0 ** -24
# FP32 roundings per product term of a promoted sum, with a factor of 8 of
# margin: the FMA of each K block into the running sum, the scale product
# fl32(s_X s_W), and the roundings inside the tensor core's 128-wide partial
ROUNDINGS = lambda kb: 8.0 * (kb + 8)


def f64(t):
    return t.detach().to("cpu").double().numpy()


def assert_close(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    err = np.abs(gpu - ref)
    bound = RTOL * np.abs(ref) + ATOL_RMS * rms
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"worst at {i}: gpu={gpu[i]} ref={ref[i]} rms={rms}")


def accumulation_bound(xq, xs, w, G, U):
    """Bound on |a_kernel - a| for a = silu(G) * U of FP8 rows (xq, xs) and
    expert w: the sums G and U are promoted over d/128 K blocks in FP32, so
    each is off by at most ROUNDINGS * 2^-24 * (sum of |products|); the
    error carries through silu (|silu'| <= 1.1) and the product, plus the
    kernel's own roundings of silu and the product."""
    A = np.abs(O.dequant_1x128(xq, xs))
    kb = A.shape[1] // 128
    dG = ROUNDINGS(kb) * EPS32 * (A @ np.abs(O.dequant_128x128(w["gate_q"], w["gate_s"])).T)
    dU = ROUNDINGS(kb) * EPS32 * (A @ np.abs(O.dequant_128x128(w["up_q"], w["up_s"])).T)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-G))
    silu = G * sig
    dsilu = np.minimum(np.abs(sig * (1.0 + G * (1.0 - sig))), 1.1)
    return dsilu * dG * np.abs(U) + np.abs(silu) * dU + 8 * EPS32 * np.abs(silu * U)


def near_tie_rows(hq_gpu, hs_gpu, a32, da, hq_ref, hs_ref, what):
    """Checks the kernel's intermediate (codes hq_gpu [R, I], scales hs_gpu
    [R, I/128]) against the oracle's (a32, hq_ref, hs_ref) under the rule
    above, da being accumulation_bound for the same rows. Returns the rows
    holding an accepted different code, and the largest ratio of an accepted
    element's distance to its rounding boundary over its bound."""
    hq_gpu = np.asarray(hq_gpu, np.uint8)
    hs_gpu = np.asarray(hs_gpu, np.float64)
    srel = np.abs(hs_gpu / hs_ref - 1.0)
    assert srel.max(initial=0.0) <= SCALE_RTOL, f"{what}: scale off by {srel.max()}"
    diff = hq_gpu != hq_ref
    if not diff.any():
        return np.zeros(0, np.int64), 0.0
    r, c = np.nonzero(diff)
    blk = c // 128
    x = a32[r, c] / hs_ref[r, blk]
    dx = da[r, c] / hs_ref[r, blk] + np.abs(x) * (srel[r, blk] + 4 * EPS32)
    lo, hi = decode(encode(x - dx)), decode(encode(x + dx))
    vg = decode(hq_gpu[r, c])
    ok = (vg >= lo) & (vg <= hi)
    assert ok.all(), (f"{what}: {int((~ok).sum())} codes outside the accumulation bound; first at row "
                      f"{r[~ok][0]} col {c[~ok][0]}: x={x[~ok][0]} bound {dx[~ok][0]} gpu value {vg[~ok][0]}")
    frac = diff.mean()
    assert frac <= 1e-3, f"{what}: {frac:.3g} of the intermediate codes differ"
    # how close to its boundary each accepted element was, in units of its bound
    vo = decode(hq_ref[r, c])
    ratio = np.abs(x - 0.5 * (vg + vo)) / np.maximum(dx, 1e-300)
    return np.unique(r), float(ratio.max())


def down_bound(hq, hs, w):
    """Bound on |y_kernel - y| for the down projection y = H W_down^T of FP8
    intermediate rows (hq, hs): I/128 K blocks promoted in FP32."""
    H = np.abs(O.dequant_1x128(hq, hs))
    kb = H.shape[1] // 128
    return ROUNDINGS(kb) * EPS32 * (H @ np.abs(O.dequant_128x128(w["down_q"], w["down_s"])).T)


def assert_bf16_rounding(gpu, ref, bound, what):
    """gpu: the kernel's bf16 outputs (as float64); ref: the oracle's float64
    values; bound: how far the kernel's FP32 sums can be from ref. Each output
    must be a bf16 rounding of some value within the bound. Returns the number
    of outputs that took the other side of a bf16 midpoint."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    lo, hi, mid = round_bf16(ref - bound), round_bf16(ref + bound), round_bf16(ref)
    bad = (gpu < lo) | (gpu > hi)
    if bad.any():
        i = np.unravel_index(np.argmax(bad), bad.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outputs are no bf16 rounding of the "
                             f"oracle's value within the accumulation bound; first at {i}: gpu={gpu[i]} "
                             f"ref={ref[i]} bound={np.broadcast_to(bound, ref.shape)[i]}")
    return int((gpu != mid).sum())
