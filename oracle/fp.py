"""Floating-point rounding steps used by the quantizers, written from their definitions.

TEST INFRASTRUCTURE (oracle): see the package docstring.

The quantizers divide and subtract in IEEE binary32 with round-to-nearest-even and
store some values in binary16.  NumPy's float32 and float16 arithmetic is IEEE, so these
helpers are thin; each is pinned in tests/test_oracle_fp.py against exact rational
arithmetic (``fractions.Fraction``) so that a wrong rounding would be caught.

E4M3 follows the OCP 8-bit floating point specification's "E4M3FN" encoding (the pages
name E4M3 in [P-vLLM] "KV Cache量化策略：INT8与FP8精度对比与选择" but define no bits):
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, the all-ones
pattern S.1111.111 is NaN, largest finite magnitude 448, subnormals m/8 * 2**-6.
"""

import numpy as np

E4M3_MAX = 448.0


def f32(x):
    """Round to the nearest binary32 value (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f16(x):
    """Round binary32 values to the nearest binary16 value (ties to even)."""
    return np.asarray(x, dtype=np.float32).astype(np.float16)


def div32(a, b):
    """IEEE binary32 quotient a / b, rounded to nearest-even (a, b binary32)."""
    a = np.asarray(a, dtype=np.float32)
    b = np.asarray(b, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.divide(a, b, dtype=np.float32)


def sub32(a, b):
    """IEEE binary32 difference a - b, rounded to nearest-even."""
    return np.subtract(np.asarray(a, np.float32), np.asarray(b, np.float32), dtype=np.float32)


def round_half_even(x):
    """Round to the nearest integer, ties to the even integer (torch.round's rule)."""
    return np.rint(np.asarray(x))


# ----------------------------------------------------------------------------- E4M3
def e4m3_decode_table():
    """float64 value of each of the 256 E4M3FN codes (NaN for 0x7F and 0xFF)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if (c >> 7) & 1 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_decode_table()
# The 127 finite non-negative magnitudes, indexed by their code 0x00..0x7E (increasing).
_E4M3_POS = _E4M3[:127].copy()


def e4m3_decode(codes):
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(r):
    """Encode finite binary32 values r as E4M3FN codes.

    The magnitude goes to the nearest finite E4M3 magnitude; an exact tie goes to the
    code with the even mantissa (even code); magnitudes above 448 saturate to 448
    (0x7E).  The sign bit is the sign of r, also when the magnitude rounds to zero.
    The 127 magnitudes increase with the code, so the nearest one is one of the two
    neighbours of |r| in that sorted list; the tie rule picks the even one of the two
    (adjacent codes, so exactly one is even).
    """
    r = np.asarray(r, dtype=np.float32)
    flat = r.reshape(-1).astype(np.float64)
    # saturation first: a magnitude beyond 448 encodes as 448
    a = np.minimum(np.abs(flat), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 126)   # first >= a
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    even = np.where(lo % 2 == 0, lo, hi)
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, even))
    out = pick.astype(np.uint8)
    out[np.signbit(flat)] |= 0x80
    return out.reshape(r.shape)


# ----------------------------------------------------------------------------- bf16
def bf16_bits(x):
    """uint16 bit pattern of values that are exactly representable in bfloat16."""
    x32 = np.asarray(x, dtype=np.float32)
    bits = x32.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("value not representable in bfloat16")
    return (bits >> 16).astype(np.uint16)


def bf16_value(bits):
    """float64 value of bfloat16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    Used only to compare a bfloat16 output with the float64 result; it rounds in one
    step from float64 with exact integer arithmetic on the binary64 pattern.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    flat = x.reshape(-1)
    o = out.reshape(-1)
    for i, v in enumerate(flat):
        if v == 0.0 or not np.isfinite(v):
            o[i] = v
            continue
        m, e = np.frexp(abs(v))          # v = m * 2**e, 0.5 <= m < 1
        e = max(e, -125)                 # bf16 subnormals share the min exponent
        scale = 2.0 ** (8 - e)           # 8 significant bits
        t = abs(v) * scale               # exact (power-of-two scaling)
        r = np.rint(t)                   # ties to even
        o[i] = np.copysign(r / scale, v)
    return out


def f16_value(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64)
