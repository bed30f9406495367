"""Test-side number formats, written from the format definitions.

Independent of the oracle's C codecs: value tables are enumerated code by
code from (sign, exponent, fraction), and encoding is a nearest-value search
over the sorted table with an exact midpoint comparison (ties to the code
with the even fraction LSB), saturating at the largest finite magnitude.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# name: (exponent bits, fraction bits, bias, has_inf, nan_allones)
FORMATS = {
    "e4m3": (4, 3, 7, False, True),
    "e5m2": (5, 2, 15, True, False),
    "e2m1": (2, 1, 1, False, False),
}


def code_value(fmt: str, code: int) -> float:
    E, M, B, has_inf, nan_allones = FORMATS[fmt]
    s = (code >> (E + M)) & 1
    e = (code >> M) & ((1 << E) - 1)
    m = code & ((1 << M) - 1)
    if has_inf and e == (1 << E) - 1:
        v = float("inf") if m == 0 else float("nan")
    elif nan_allones and e == (1 << E) - 1 and m == (1 << M) - 1:
        v = float("nan")
    elif e == 0:
        v = m / (1 << M) * 2.0 ** (1 - B)
    else:
        v = (1 + m / (1 << M)) * 2.0 ** (e - B)
    return -v if s else v


def positive_table(fmt: str):
    """(codes, values) of the finite non-negative codes, sorted by value."""
    E, M, _, _, _ = FORMATS[fmt]
    codes = []
    vals = []
    for c in range(1 << (E + M)):
        v = code_value(fmt, c)
        if np.isfinite(v):
            codes.append(c)
            vals.append(v)
    order = np.argsort(vals, kind="stable")
    return np.array(codes)[order], np.array(vals, dtype=np.float64)[order]


def max_finite(fmt: str) -> float:
    return float(positive_table(fmt)[1][-1])


def nearest_code(fmt: str, v) -> np.ndarray:
    """Round-to-nearest-even, saturating, sign kept (including -0)."""
    E, M, _, _, _ = FORMATS[fmt]
    v = np.asarray(v, dtype=np.float64).ravel()
    codes, vals = positive_table(fmt)
    a = np.abs(v)
    hi = np.searchsorted(vals, a, side="left")
    hi_c = np.minimum(hi, len(vals) - 1)
    lo_c = np.maximum(hi - 1, 0)
    exact = vals[hi_c] == a
    mid = (vals[lo_c] + vals[hi_c]) / 2.0          # exact: both dyadic and small
    pick_lo = a < mid
    pick_hi = a > mid
    tie = ~(pick_lo | pick_hi)
    even_lo = (codes[lo_c] & 1) == 0
    choice = np.where(pick_lo, lo_c, np.where(pick_hi, hi_c, np.where(even_lo, lo_c, hi_c)))
    choice = np.where(exact, hi_c, choice)
    choice = np.where(a >= vals[-1], len(vals) - 1, choice)
    out = codes[choice].astype(np.uint32)
    sign = np.signbit(v).astype(np.uint32) << (E + M)
    return out | sign


def decode(fmt: str, codes) -> np.ndarray:
    table = np.array([code_value(fmt, c) for c in range(1 << (sum(FORMATS[fmt][:2]) + 1))])
    return table[np.asarray(codes, dtype=np.int64)]


def bf16_value(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint32) << 16
    return b.astype(np.uint32).view(np.float32)


def e8m0_value(b: int) -> Fraction:
    return Fraction(2) ** (b - 127)


def exact(v) -> Fraction:
    return Fraction(float(v))


def nearest_within(fmt: str, r, codes, slack_rel: float = 2.0 ** -22) -> np.ndarray:
    """True where code is a correct rounding of the real value r up to a relative slack.

    A code passes when its value is the nearest grid point to r, or -- only when r lies
    within slack_rel*|r| of the midpoint of its two neighbours -- the other neighbour
    (this absorbs the binary32 rounding of r itself).  Beyond the largest finite value
    the code must be the saturated one.  The sign bit must equal the sign of r.
    """
    E, M, _, _, _ = FORMATS[fmt]
    r = np.asarray(r, dtype=np.float64).ravel()
    codes = np.asarray(codes, dtype=np.int64).ravel()
    mag_codes = codes & ((1 << (E + M)) - 1)
    vals = np.abs(decode(fmt, mag_codes).astype(np.float64))
    _, table = positive_table(fmt)
    a = np.abs(r)
    m = table[-1]
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    lo_v, hi_v = table[lo], table[hi]
    exact_hit = hi_v == a
    mid = (lo_v + hi_v) / 2.0
    near_mid = np.abs(a - mid) <= slack_rel * a
    nearest = np.where(a < mid, lo_v, hi_v)
    ok = (vals == nearest) | (near_mid & ((vals == lo_v) | (vals == hi_v)))
    ok = np.where(exact_hit, vals == a, ok)
    sat = a >= m * (1 + slack_rel)
    ok = np.where(sat, vals == m, ok)
    ok = np.where((a >= m) & ~sat, (vals == m) | ok, ok)
    sign_ok = ((codes >> (E + M)) & 1) == np.signbit(r).astype(np.int64)
    return ok & sign_ok
