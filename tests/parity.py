"""Parity helpers shared by the GPU tests.

Tolerance for floating-point outputs: |gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref).

Requantisation near-ties. The expert intermediate a = silu(G) * U is
accumulated by the kernel in FP32 (each 128-wide K block promoted in FP32) and
by the oracle in float64, so the two differ by FP32 rounding. Its E4M3 code
(1x128 tiles along I) is an integer decided by floating point: where the
oracle's value x = a / scale lies within a relative NEAR_TIE of the rounding
boundary between two adjacent E4M3 values, either code is a valid outcome of
the method. The kernel's intermediate codes must then equal the oracle's
everywhere else, its tile scales must agree to SCALE_RTOL, and a row with an
accepted near-tie code is re-evaluated by the oracle's down projection on the
kernel's codes (as a token whose top-K keys tie within the routing margin is
evaluated under the kernel's selection) before its output is compared.
"""
import numpy as np

from oracle.e4m3 import decode

RTOL, ATOL_RMS = 8e-3, 1e-3
NEAR_TIE = 1e-4          # relative distance of x to the rounding boundary
SCALE_RTOL = 1e-4        # tile scales fl32(amax / 448): amax accumulated in FP32 vs float64


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


def near_tie_rows(hq_gpu, hs_gpu, a32, hq_ref, hs_ref, what):
    """Checks the kernel's intermediate (codes hq_gpu [R, I], scales hs_gpu
    [R, I/128]) against the oracle's (a32, hq_ref, hs_ref) under the
    near-tie rule; returns the rows holding an accepted near-tie code, and
    the largest relative distance to the boundary seen among them."""
    hq_gpu = np.asarray(hq_gpu, np.uint8)
    hs_gpu = np.asarray(hs_gpu, np.float64)
    srel = np.abs(hs_gpu / hs_ref - 1.0)
    assert srel.max(initial=0.0) <= SCALE_RTOL, f"{what}: scale off by {srel.max()}"
    diff = hq_gpu != hq_ref
    if not diff.any():
        return np.zeros(0, np.int64), 0.0
    r, c = np.nonzero(diff)
    g, o = hq_gpu[r, c].astype(np.int64), hq_ref[r, c].astype(np.int64)
    # adjacent codes: same sign, magnitudes one step apart (E4M3 magnitudes
    # are monotonic in the code's low 7 bits); +-0 count as equal magnitude
    mg, mo = g & 0x7F, o & 0x7F
    same_sign = ((g ^ o) & 0x80) == 0
    adjacent = (np.abs(mg - mo) == 1) & (same_sign | (np.minimum(mg, mo) == 0))
    assert adjacent.all(), (f"{what}: {int((~adjacent).sum())} codes more than one step apart, "
                            f"first at row {r[~adjacent][0]} col {c[~adjacent][0]}")
    x = a32[r, c] / hs_ref[r, c // 128]
    m = 0.5 * (decode(g) + decode(o))
    dist = np.abs(x - m) / np.maximum(np.abs(m), 2.0 ** -9)
    assert (dist <= NEAR_TIE).all(), (f"{what}: a code differs away from a rounding boundary "
                                      f"(relative distance {dist.max():.3g}, row {r[np.argmax(dist)]})")
    frac = diff.mean()
    assert frac <= 1e-3, f"{what}: {frac:.3g} of the intermediate codes differ"
    return np.unique(r), float(dist.max())
