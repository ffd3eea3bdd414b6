"""Number formats used by the oracle: FP8 E4M3, bfloat16, float32.

Test infrastructure only (see the package docstring).

E4M3 is the FP8 format the method uses for every FP8 tensor ("DeepSeek-V3
Teknik Raporu", Temel fikirler, bullet "FP8 Karma Duyarlıklı Eğitim": "Tüm
tensörlerde E4M3 kullanır"). The pages name the format only; its bit layout is
the public OCP 8-bit floating point definition:

  * 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
  * exponent field e = 1..15: value 2^(e-7) * (1 + m/8);
  * exponent field e = 0:     value 2^-6 * (m/8)   (subnormals, and zero);
  * S.1111.111 (0x7F, 0xFF) is NaN; there are no infinities;
  * the largest finite magnitude is 1.1110 * 2^8 = 448 (code 0x7E).

Encoding rounds to the nearest representable value, ties to the even
mantissa, and saturates magnitudes above 448 to 448 ("satfinite").

All functions take and return float64 numpy arrays.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_MIN_SUBNORMAL = 2.0 ** -9


def decode_table() -> np.ndarray:
    """Value of each of the 256 codes (NaN for 0x7F and 0xFF)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (2.0 ** -6) * (m / 8.0)
        else:
            vals[code] = sign * (2.0 ** (e - 7)) * (1.0 + m / 8.0)
    return vals


_TABLE = decode_table()


def decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float64 values."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def encode(x: np.ndarray) -> np.ndarray:
    """float64 values -> uint8 E4M3 codes, round-to-nearest-even, satfinite.

    Within the binade [2^k, 2^(k+1)) (k >= -6) the representable magnitudes are
    n * 2^(k-3) with n = 8..15 (exponent field k+7, mantissa n-8); below 2^-6
    they are the subnormals n * 2^-9, n = 0..7 (exponent field 0, mantissa n).
    So the nearest value has n = rint(|x| / 2^(k-3)); numpy's rint rounds ties
    to the even integer, and n's parity is the mantissa's parity. n = 16 is the
    carry into the next binade (mantissa 0, also even); n = 8 from the
    subnormal range is the smallest normal.
    """
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN input to the E4M3 encoder")
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)              # satfinite
    _, ex = np.frexp(a)                              # a = f * 2^ex, f in [0.5, 1)
    k = np.maximum(ex - 1, -6)                       # binade; the subnormals share 2^-9
    n = np.rint(np.ldexp(a, 3 - k))                  # a / 2^(k-3), exact scaling, RNE
    carry = n >= 16.0
    k = np.where(carry, k + 1, k)
    n = np.where(carry, 8.0, n).astype(np.int64)
    sub = n < 8                                      # only when k == -6
    efield = np.where(sub, 0, k + 7).astype(np.int64)
    mfield = np.where(sub, n, n - 8)
    code = (efield << 3) | mfield | (neg.astype(np.int64) << 7)
    return code.astype(np.uint8)


def round_fp32(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest float32 (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even).

    bfloat16 keeps 8 significant bits and float32's exponent range: inside
    [2^k, 2^(k+1)) the spacing is 2^(k-7); below 2^-126 the subnormal spacing
    is 2^-133. Values beyond the finite range do not occur in this layer.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)
    k = np.maximum(ex.astype(np.int64) - 1, -126)
    q = np.ldexp(1.0, k - 7)
    r = np.rint(a / q) * q
    return np.copysign(r, x)
