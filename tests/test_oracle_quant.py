"""Pins of the oracle quantizers: exact arithmetic, brute force, closed forms."""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp, quant
from tests.test_oracle_fp import exact_round


def _rhe(fr):
    """Round a Fraction to the nearest integer, ties to even."""
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


# ----------------------------------------------------------------------------- INT8
@pytest.mark.parametrize("scale_bits", [0x3C000000, 0x3D0A3D71, 0x3E8F5C29, 0x3F800000])
def test_int8_bruteforce_over_all_fp16_values(scale_bits):
    """Every finite fp16 x against the exact two-step definition (binary32 quotient,
    then round half even, then clamp), for several scales."""
    s = np.array([scale_bits], np.uint32).view(np.float32)[0]
    x = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16)
    x = x[np.isfinite(x)].astype(np.float32)
    q = quant.int8_quantize(x, np.float32(s))
    sf = Fraction(float(s))
    for xi, qi in zip(x[::7], q[::7]):
        r = exact_round(Fraction(float(xi)) / sf, 24, -126)
        want = max(-128, min(127, _rhe(r)))
        assert int(qi) == want, (xi, s, qi, want)


def test_int8_dynamic_scale_closed_form():
    rows = np.array([[127.0, -3.0, 0.5], [-2.0, 1.0, 0.0], [0.0, 0.0, 0.0]], np.float32)
    s = quant.int8_scale_dynamic(rows)
    assert s[0] == np.float32(1.0)
    assert Fraction(float(s[1])) == exact_round(Fraction(2) / 127, 24, -126)
    assert s[2] == 0.0
    q = quant.int8_quantize(rows, s)
    np.testing.assert_array_equal(q[0], [127, -3, 0])      # 0.5 -> 0 (half to even)
    np.testing.assert_array_equal(q[2], [0, 0, 0])          # zero row: no division


def test_int8_grid_exact_special_case():
    """x = k * 2^-e with one element +-127 * 2^-e: s = 2^-e exactly and q = k."""
    rng = np.random.default_rng(0)
    for e in (-3, 0, 5, 9):
        k = rng.integers(-127, 128, size=(50, 64))
        k[:, 0] = rng.choice([-127, 127], size=50)
        x = (k * 2.0 ** -e).astype(np.float32)
        s = quant.int8_scale_dynamic(x)
        assert np.all(s == np.float32(2.0 ** -e))
        np.testing.assert_array_equal(quant.int8_quantize(x, s), k)
        np.testing.assert_array_equal(quant.int8_dequantize(quant.int8_quantize(x, s), s), x)


def test_int8_round_trip_bound():
    """|x - q s| <= s (1/2 + 2^-17) when nothing clamps: the quotient, below 128 in
    magnitude, is rounded to binary32 (half an ulp <= 2^-17) before the integer rounding."""
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(400, 128, generator=g) * 3).to(torch.bfloat16).float().numpy()
    s = quant.int8_scale_dynamic(x)
    q = quant.int8_quantize(x, s)
    err = np.abs(x.astype(np.float64) - quant.int8_dequantize(q, s))
    bound = s.astype(np.float64)[:, None] * (0.5 + 2.0 ** -17)
    assert np.all(err <= bound)
    assert np.all(np.abs(q.astype(int)) <= 127)


def test_int8_static_scale_clamps():
    x = np.array([[1000.0, -1000.0, 1.0, -129.0]], np.float32)
    q = quant.int8_quantize(x, np.array([1.0], np.float32))
    np.testing.assert_array_equal(q, [[127, -128, 1, -128]])


# ----------------------------------------------------------------------------- FP8
def test_fp8_power_of_two_scale_exact_round_trip():
    t = fp.e4m3_decode_table()
    finite = t[np.isfinite(t)]
    for e in (-4, 0, 3):
        s = np.float32(2.0 ** e)
        x = (finite * 2.0 ** e).astype(np.float32)[None, :]
        c = quant.fp8_quantize(x, np.array([s]))
        np.testing.assert_array_equal(quant.fp8_dequantize(c, np.array([s]))[0], x[0].astype(np.float64))


def test_fp8_calibration_and_saturation():
    g = torch.Generator().manual_seed(3)
    w = torch.randn(256, 4, 128, generator=g).to(torch.bfloat16).float().numpy()
    s = quant.fp8_calibrate(w)
    for h in range(4):
        m = np.max(np.abs(w[:, h, :]))
        assert Fraction(float(s[h])) == exact_round(Fraction(float(m)) / 448, 24, -126)
    # a value twice the warm-up max saturates to +-448 * s
    x = np.array([[2 * np.max(np.abs(w[:, 0, :])), -2 * np.max(np.abs(w[:, 0, :]))]], np.float32)
    c = quant.fp8_quantize(x, s[:1])
    np.testing.assert_array_equal(c, [[0x7E, 0xFE]])


def test_head_calibration_exact_and_int8_static_round_trip():
    """Per-head static scale: max over tokens and channels of |x| / qmax, one binary32
    rounding of the exact quotient; with qmax 127 the warm-up's largest value gets code
    +-127 exactly and every warm-up value stays inside the clamp."""
    g = torch.Generator().manual_seed(4)
    w = torch.randn(256, 3, 128, generator=g).to(torch.bfloat16).float().numpy()
    for qmax in (127.0, 448.0):
        s = quant.head_calibrate(w, qmax)
        assert s.shape == (3,) and s.dtype == np.float32
        for h in range(3):
            m = np.max(np.abs(w[:, h, :]))
            assert Fraction(float(s[h])) == exact_round(Fraction(float(m)) / Fraction(qmax), 24, -126)
    np.testing.assert_array_equal(quant.head_calibrate(w, 448.0), quant.fp8_calibrate(w))
    s = quant.head_calibrate(w, 127.0)
    for h in range(3):
        c = quant.int8_quantize(w[:, h, :].reshape(1, -1), s[h:h + 1])
        assert np.max(np.abs(c.astype(np.int64))) == 127
    # an all-zero head gives scale 0
    z = np.zeros((8, 2, 64), np.float32)
    np.testing.assert_array_equal(quant.head_calibrate(z, 127.0), [0.0, 0.0])


def test_fp8_quantize_is_nearest_code():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(64, 128, generator=g).to(torch.bfloat16).float().numpy()
    s = quant.fp8_scale_dynamic(x)
    c = quant.fp8_quantize(x, s)
    r = fp.div32(x, s[:, None]).astype(np.float64)
    t = fp.e4m3_decode_table()
    fin = np.where(np.isnan(t), np.inf, t)
    got = fp.e4m3_decode(c)
    best = np.min(np.abs(r[..., None] - fin[None, None, :]), axis=-1)
    np.testing.assert_array_equal(np.abs(r - got), best)


# ----------------------------------------------------------------------------- INT4
def test_int4_nearest_code_bruteforce():
    """Each code minimises |x - (c - z) s| over the 16 codes, given the stored (s, z)."""
    g = torch.Generator().manual_seed(7)
    for trial in range(40):
        x = (torch.randn(64, generator=g) * (0.1 + trial)).to(torch.bfloat16).float().numpy()
        if trial % 5 == 0:
            x = np.abs(x)                      # all positive: range widened to 0
        c, s, z = quant.int4_quantize_group(x)
        assert 0 <= float(z) <= 15 and float(z) == int(float(z))
        grid = (np.arange(16) - np.float64(z)) * np.float64(s)
        d = np.abs(x.astype(np.float64)[:, None] - grid[None, :])
        chosen = d[np.arange(64), c]
        assert np.all(chosen <= d.min(axis=1) + 1e-12 * np.abs(x).max())


def test_int4_scale_steps_exact():
    x = np.array([3.0, -1.5, 0.25, 7.75] + [0.0] * 60, np.float32)
    c, s, z = quant.int4_quantize_group(x)
    s_want = exact_round(exact_round(Fraction(775, 100) + Fraction(3, 2), 24, -126) / 15, 24, -126)
    assert Fraction(float(s)) == exact_round(s_want, 11, -14)
    z_want = max(0, min(15, _rhe(exact_round(Fraction(3, 2) / Fraction(float(s)), 24, -126))))
    assert float(z) == z_want


def test_int4_grid_exact_round_trip():
    """Values on the grid (k - z0) 2^-e spanning all 16 codes round-trip exactly."""
    rng = np.random.default_rng(9)
    for e in (-6, -2, 0, 3):
        for z0 in (0, 4, 15):
            k = rng.integers(0, 16, 64)
            k[0], k[1] = 0, 15
            x = ((k - z0) * 2.0 ** -e).astype(np.float32)
            c, s, z = quant.int4_quantize_group(x)
            assert float(s) == 2.0 ** -e and float(z) == z0
            np.testing.assert_array_equal(c, k)
            np.testing.assert_array_equal(quant.int4_dequantize(c, s, z), x.astype(np.float64))


def test_int4_constant_and_zero_groups():
    c, s, z = quant.int4_quantize_group(np.zeros(64, np.float32))
    assert float(s) == 0 and float(z) == 0 and not c.any()
    # a constant group: the range is [x, 0]; the fp16 scale is within half an fp16 ulp
    # of x/15, so the reconstruction is within 15 * s * 2^-11 of x
    c, s, z = quant.int4_quantize_group(np.full(64, -2.0, np.float32))
    assert float(z) == 15 and not c.any()
    err = np.abs(quant.int4_dequantize(c, s, z) + 2.0)
    assert np.all(err <= 15 * float(s) * 2.0 ** -11)
    # a grid-exact constant (-15 * 2^-3) reconstructs exactly
    c, s, z = quant.int4_quantize_group(np.full(64, -15 * 2.0 ** -3, np.float32))
    np.testing.assert_array_equal(quant.int4_dequantize(c, s, z), np.full(64, -15 * 2.0 ** -3))


def test_int4_round_trip_bound():
    g = torch.Generator().manual_seed(13)
    x = torch.randn(64, 128, generator=g).to(torch.bfloat16).float().numpy()
    codes, s, z = quant.int4_keys_block(x)
    deq = (codes.astype(np.float64) - z.astype(np.float64)) * s.astype(np.float64)
    # s is rounded to fp16 (rel. 2^-11): the grid may fall short of the range by 15 s 2^-11
    bound = s.astype(np.float64) * (0.5 + 15 * 2.0 ** -11) + 1e-12
    assert np.all(np.abs(x - deq) <= bound[None, :])


def test_nibble_packing():
    c = np.array([1, 2, 15, 0, 7, 8], np.uint8)
    p = quant.pack_nibbles(c)
    np.testing.assert_array_equal(p, [0x21, 0x0F, 0x87])
    np.testing.assert_array_equal(quant.unpack_nibbles(p), c)


def test_kivi_axes():
    """Keys group over tokens (per channel), values over channels (per token)."""
    rng = np.random.default_rng(2)
    k = rng.standard_normal((64, 128)).astype(np.float32)
    k[:, 5] *= 100.0                              # one outlier channel
    kc, ks, kz = quant.int4_keys_block(k)
    assert ks.shape == (128,) and ks[5] > 50 * np.median(ks)
    v = rng.standard_normal(128).astype(np.float32)
    v[70] = 1000.0                                # outlier only in the second group
    vc, vs, vz = quant.int4_values_row(v)
    assert vs.shape == (2,) and vs[1] > 100 * vs[0]


# ------------------------------------------------- INT4 with a float zero point (group min)
def test_int4_float_zero_nearest_code_bruteforce():
    """Each code minimises |x - (c s + m)| over the 16 codes, given the stored (s, m)."""
    g = torch.Generator().manual_seed(17)
    for trial in range(40):
        x = (torch.randn(64, generator=g) * (0.1 + trial) + (trial % 7 - 3)).to(torch.bfloat16)
        x = x.float().numpy()
        c, s, m = quant.int4_quantize_groups_float_zero(x[None])
        c, s, m = c[0], s[0], m[0]
        grid = np.arange(16) * np.float64(s) + np.float64(m)
        d = np.abs(x.astype(np.float64)[:, None] - grid[None, :])
        chosen = d[np.arange(64), c]
        assert np.all(chosen <= d.min(axis=1) + 2.0 ** -20 * float(s))


def test_int4_float_zero_steps_exact():
    """s = fp16(fp32((hi - lo) / 15)) and m = fp16(lo), in exact arithmetic; the range is
    not widened to include 0 (an all-positive group keeps its own minimum)."""
    x = np.array([3.0, 1.5, 2.25, 7.75] + [2.0] * 60, np.float32)
    c, s, m = quant.int4_quantize_groups_float_zero(x[None])
    s_want = exact_round(exact_round(Fraction(775, 100) - Fraction(3, 2), 24, -126) / 15, 24, -126)
    assert Fraction(float(s[0])) == exact_round(s_want, 11, -14)
    assert float(m[0]) == 1.5
    assert c[0][1] == 0 and c[0][3] == 15
    want2 = _rhe(exact_round(Fraction(1, 2) / Fraction(float(s[0])), 24, -126))   # x = 2.0
    assert c[0][4] == want2


def test_int4_float_zero_grid_exact_round_trip():
    """Values on the grid m0 + k 2^-e (all 16 codes used, m0 on both sides of 0) come back
    exactly."""
    rng = np.random.default_rng(19)
    for e in (-3, 0, 2, 5):
        for m0 in (-5.0, -0.75, 0.0, 1.25, 9.0):
            k = rng.integers(0, 16, 64)
            k[0], k[1] = 0, 15
            x = (m0 + k * 2.0 ** -e).astype(np.float32)
            c, s, m = quant.int4_quantize_groups_float_zero(x[None])
            assert float(s[0]) == 2.0 ** -e and float(m[0]) == m0
            np.testing.assert_array_equal(c[0], k)
            np.testing.assert_array_equal(quant.int4_dequantize_float_zero(c[0], s[0], m[0]),
                                          x.astype(np.float64))


def test_int4_float_zero_constant_group_and_bound():
    c, s, m = quant.int4_quantize_groups_float_zero(np.full((1, 64), -2.5, np.float32))
    assert float(s[0]) == 0 and float(m[0]) == -2.5 and not c.any()
    np.testing.assert_array_equal(quant.int4_dequantize_float_zero(c[0], s[0], m[0]), -2.5)
    g = torch.Generator().manual_seed(23)
    x = (torch.randn(128, 64, generator=g) + 3.0).to(torch.bfloat16).float().numpy()
    c, s, m = quant.int4_quantize_groups_float_zero(x)
    deq = quant.int4_dequantize_float_zero(c, s[:, None], m[:, None])
    s64 = s.astype(np.float64)[:, None]
    # m is a bf16 value, exact in fp16; s is rounded to fp16 (rel. 2^-11)
    assert np.all(np.abs(x - deq) <= s64 * (0.5 + 15 * 2.0 ** -11) + 1e-12)


def test_int4_per_token_keys_group_like_values():
    """The per-token variant groups each key row over 64-channel runs: an outlier channel
    raises only its own group's scale, for every token alike."""
    rng = np.random.default_rng(29)
    k = rng.standard_normal((64, 128)).astype(np.float32)
    k[:, 5] = 500.0
    c, s, z = quant.int4_values_row(k)
    assert s.shape == (64, 2)
    assert np.all(s[:, 0] > 20 * s[:, 1])
    c1, s1, z1 = quant.int4_values_row(k[7])
    np.testing.assert_array_equal(c[7], c1)
    np.testing.assert_array_equal(s[7], s1)


# ------------------------------------------------------------------------- 2-bit
@pytest.mark.parametrize("float_zero", [False, True])
def test_int2_nearest_code_bruteforce(float_zero):
    """2-bit groups (codes 0..3): each code is a nearest grid point given the stored
    parameters, for both zero-point forms."""
    g = torch.Generator().manual_seed(31)
    for trial in range(40):
        x = (torch.randn(64, generator=g) * (0.1 + trial) + (trial % 5 - 2)).to(torch.bfloat16)
        x = x.float().numpy()
        if float_zero:
            c, s, m = quant.int4_quantize_groups_float_zero(x[None], bits=2)
            grid = np.arange(4) * np.float64(s[0]) + np.float64(m[0])
        else:
            c, s, z = quant.int4_quantize_groups(x[None], bits=2)
            assert 0 <= float(z[0]) <= 3
            grid = (np.arange(4) - np.float64(z[0])) * np.float64(s[0])
        d = np.abs(x.astype(np.float64)[:, None] - grid[None, :])
        chosen = d[np.arange(64), c[0]]
        assert c.max() <= 3
        assert np.all(chosen <= d.min(axis=1) + 2.0 ** -20 * float(s[0]))


def test_int2_steps_exact():
    """s = fp16(fp32((hi - lo) / 3)), z = RNE(-lo / s) in exact arithmetic."""
    x = np.array([3.0, -1.5, 0.25, 2.0] + [0.0] * 60, np.float32)
    c, s, z = quant.int4_quantize_groups(x[None], bits=2)
    s_want = exact_round(exact_round(Fraction(3) + Fraction(3, 2), 24, -126) / 3, 24, -126)
    assert Fraction(float(s[0])) == exact_round(s_want, 11, -14)
    z_want = max(0, min(3, _rhe(exact_round(Fraction(3, 2) / Fraction(float(s[0])), 24, -126))))
    assert float(z[0]) == z_want == 1
    assert list(c[0][:4]) == [3, 0, 1, 2]


def test_int2_grid_exact_round_trip():
    rng = np.random.default_rng(37)
    for e in (-2, 0, 3):
        for z0 in (0, 1, 3):
            k = rng.integers(0, 4, 64)
            k[0], k[1] = 0, 3
            x = ((k - z0) * 2.0 ** -e).astype(np.float32)
            c, s, z = quant.int4_quantize_groups(x[None], bits=2)
            assert float(s[0]) == 2.0 ** -e and float(z[0]) == z0
            np.testing.assert_array_equal(c[0], k)
        m0 = -1.25
        x = (m0 + k * 2.0 ** -e).astype(np.float32)
        c, s, m = quant.int4_quantize_groups_float_zero(x[None], bits=2)
        assert float(s[0]) == 2.0 ** -e and float(m[0]) == m0
        np.testing.assert_array_equal(c[0], k)


def test_crumb_packing():
    c = np.array([1, 2, 3, 0, 3, 3, 0, 1], np.uint8)
    p = quant.pack_codes(c, 2)
    np.testing.assert_array_equal(p, [0b00111001, 0b01001111])
    np.testing.assert_array_equal(quant.unpack_codes(p, 2), c)
    np.testing.assert_array_equal(quant.pack_codes(c, 4), quant.pack_nibbles(c))
