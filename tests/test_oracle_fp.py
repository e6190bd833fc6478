"""Pins of the oracle's rounding steps against exact rational arithmetic and torch casts."""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp


def exact_round(fr, mant_bits, emin):
    """Nearest value with `mant_bits` significand bits (min normal exponent emin), ties even.

    Exact integer arithmetic on a Fraction; overflow is not modelled.
    """
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - (mant_bits - 1))
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def _rand_f32(rng, n, lo_exp=-140, hi_exp=60):
    m = rng.uniform(1.0, 2.0, n)
    e = rng.integers(lo_exp, hi_exp, n)
    s = rng.choice([-1.0, 1.0], n)
    return (s * m * np.exp2(e)).astype(np.float32)


def test_div32_matches_exact_binary32_rounding():
    rng = np.random.default_rng(1)
    a = _rand_f32(rng, 4000)
    b = _rand_f32(rng, 4000, -40, 40)
    q = fp.div32(a, b)
    for ai, bi, qi in zip(a, b, q):
        want = exact_round(Fraction(float(ai)) / Fraction(float(bi)), 24, -126)
        if abs(want) > Fraction(float(np.finfo(np.float32).max)):
            continue
        assert Fraction(float(qi)) == want, (ai, bi, qi, float(want))


def test_div32_int8_style_quotients():
    # x / (m / 127) for bf16-like x: the exact path the INT8 quantizer takes
    rng = np.random.default_rng(2)
    x = torch.randn(3000, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).float().numpy()
    m = np.float32(np.max(np.abs(x)))
    s = fp.div32(m, np.float32(127.0))
    assert Fraction(float(s)) == exact_round(Fraction(float(m)) / 127, 24, -126)
    r = fp.div32(x, s)
    for xi, ri in zip(x[:500], r[:500]):
        assert Fraction(float(ri)) == exact_round(Fraction(float(xi)) / Fraction(float(s)), 24, -126)
    del rng


def test_sub32_exact():
    rng = np.random.default_rng(4)
    a = _rand_f32(rng, 2000, -20, 20)
    b = _rand_f32(rng, 2000, -20, 20)
    d = fp.sub32(a, b)
    for ai, bi, di in zip(a, b, d):
        assert Fraction(float(di)) == exact_round(Fraction(float(ai)) - Fraction(float(bi)), 24, -126)


def test_f16_rounding_exact_including_ties_and_subnormals():
    rng = np.random.default_rng(5)
    vals = list(_rand_f32(rng, 3000, -26, 15))
    # exact midpoints between neighbouring float16 values (ties -> even)
    h = np.arange(0, 0x7BFF, 37, dtype=np.uint16).view(np.float16).astype(np.float64)
    hn = (np.arange(0, 0x7BFF, 37, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    vals += list(((h + hn) / 2).astype(np.float32))
    vals = np.array(vals, np.float32)
    r = fp.f16(vals)
    for v, ri in zip(vals, r):
        want = exact_round(Fraction(float(v)), 11, -14)
        if abs(want) > 65504:
            continue
        assert Fraction(float(ri)) == want, (v, ri)


def test_round_half_even():
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 0.49999997, 126.5, 127.5, -128.5])
    np.testing.assert_array_equal(fp.round_half_even(x), [0, 2, 2, -0, -2, -2, 0, 126, 128, -128])


# ----------------------------------------------------------------------------- E4M3
def test_e4m3_decode_table_matches_torch_float8_e4m3fn():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = fp.e4m3_decode_table()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])


def test_e4m3_closed_form_points():
    t = fp.e4m3_decode_table()
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    assert t[0x38] == 1.0 and t[0x80] == 0.0 and np.signbit(t[0x80])
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])


def test_e4m3_encode_matches_exact_rounding_and_torch_in_range():
    rng = np.random.default_rng(6)
    r = list(_rand_f32(rng, 3000, -12, 9))
    t = fp.e4m3_decode_table()[:127]
    r += list(((t[:-1] + t[1:]) / 2).astype(np.float32))        # every tie
    r += list((-(t[:-1] + t[1:]) / 2).astype(np.float32))
    r = np.array([x for x in r if abs(x) <= 448.0], np.float32)
    codes = fp.e4m3_encode(r)
    # exact: 4 significand bits, min normal exponent -6
    for x, c in zip(r, codes):
        want = exact_round(Fraction(float(x)), 4, -6)
        assert Fraction(float(fp.e4m3_decode(c))) == want, (x, c)
    # library routine: torch's float32 -> float8_e4m3fn cast (round to nearest even)
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)


def test_e4m3_encode_equals_brute_force_nearest():
    """The neighbour search against the plain definition: distance to all 127
    magnitudes, nearest wins, a tie goes to the even code."""
    rng = np.random.default_rng(16)
    t = fp.e4m3_decode_table()[:127]
    r = np.concatenate([
        _rand_f32(rng, 20000, -14, 10),
        ((t[:-1] + t[1:]) / 2).astype(np.float32),
        np.nextafter(((t[:-1] + t[1:]) / 2).astype(np.float32), np.float32(0)),
        np.nextafter(((t[:-1] + t[1:]) / 2).astype(np.float32), np.float32(np.inf)),
        t.astype(np.float32), np.float32([0.0, 448.0, 464.0, 1e30])])
    r = np.concatenate([r, -r])
    a = np.minimum(np.abs(r.astype(np.float64)), 448.0)[:, None]
    dist = np.abs(a - t[None, :])
    hits = dist == dist.min(axis=1, keepdims=True)
    two = hits.sum(axis=1) > 1
    idx = np.arange(127)[None, :]
    want = np.where(two, np.argmax(hits & (idx % 2 == 0), axis=1), np.argmax(hits, axis=1))
    want = want.astype(np.uint8) | np.where(np.signbit(r), 0x80, 0).astype(np.uint8)
    np.testing.assert_array_equal(fp.e4m3_encode(r), want)


def test_e4m3_saturation_and_signed_zero():
    r = np.array([448.0, 449.0, 464.0, 500.0, 1e30, -1e30, -464.0, 2.0 ** -10,
                  3 * 2.0 ** -10, -1e-30, -0.0, 0.0], np.float32)
    np.testing.assert_array_equal(
        fp.e4m3_encode(r),
        np.array([0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x00, 0x02, 0x80, 0x80, 0x00], np.uint8))


# ----------------------------------------------------------------------------- bf16
def test_bf16_round_exact():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(2000) * np.exp2(rng.integers(-20, 20, 2000))
    r = fp.bf16_round(x)
    for xi, ri in zip(x, r):
        assert Fraction(float(ri)) == exact_round(Fraction(float(xi)), 8, -126)


@pytest.mark.parametrize("bad", [1.0 + 2.0 ** -10])
def test_bf16_bits_rejects_unrepresentable(bad):
    with pytest.raises(ValueError):
        fp.bf16_bits(np.array([bad], np.float32))
