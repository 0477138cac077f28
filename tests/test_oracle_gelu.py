"""Pins of the oracle's FFN activation X_down = bf16_rn(gelu(y)) (GELU, tanh
form, correctly rounded to bf16) and of its float64 -> bf16 rounding.

* every finite bf16 input against a 120-digit evaluation of the other closed
  form, 0.5 y (1 + tanh(u)), with the nearest bf16 value checked by exact
  comparison against both neighbours;
* the tanh form against the exact (erf) GELU it approximates;
* the one-step float64 -> bf16 rounding against the float32 path where the two
  must agree, and on values no float32 can hold;
* special values."""
import mpmath
import numpy as np
from scipy.special import erf

from oracle import w4a4_oracle as orc

mpmath.mp.dps = 120


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    y = orc.bf16_bits_to_f32(bits)
    keep = np.isfinite(y)
    return bits[keep], y[keep]


def _bf16_neighbours(bits):
    """The bf16 values just below and above the one with these bits (same sign
    convention as the value: toward -inf and toward +inf)."""
    v = float(orc.bf16_bits_to_f32(np.array([bits], np.uint16))[0])
    if v == 0.0:
        return -2.0 ** -133, 2.0 ** -133
    up = orc.bf16_bits_to_f32(np.array([bits + 1], np.uint16))[0]
    dn = orc.bf16_bits_to_f32(np.array([bits - 1], np.uint16))[0]
    lo, hi = (dn, up) if v > 0 else (up, dn)
    return float(lo), float(hi)


def test_gelu_every_bf16_is_nearest_to_120_digit_value():
    bits_in, y = _all_finite_bf16()
    got = orc.f32_to_bf16_bits(orc.gelu_bf16(y))
    half_sqrt = mpmath.sqrt(2 / mpmath.pi)
    c = mpmath.mpf("0.044715")
    tiny = mpmath.mpf(2) ** -135
    for i in range(y.size):
        yv = mpmath.mpf(float(y[i]))
        u = half_sqrt * (yv + c * yv ** 3)
        g = yv * (1 + mpmath.tanh(u)) / 2
        gb = int(got[i])
        r = float(orc.bf16_bits_to_f32(np.array([gb], np.uint16))[0])
        if abs(g) < tiny:
            # far below half the smallest bf16 subnormal: a zero of the sign of y
            assert r == 0.0 and np.signbit(r) == np.signbit(y[i]), (float(y[i]), r)
            continue
        lo, hi = _bf16_neighbours(gb)
        d = abs(g - mpmath.mpf(r))
        assert d < abs(g - mpmath.mpf(lo)) and d < abs(g - mpmath.mpf(hi)), (float(y[i]), r)


def test_tanh_form_is_close_to_erf_gelu():
    _, y = _all_finite_bf16()
    y = y[np.abs(y) <= 30]
    g = orc.gelu_bf16(y).astype(np.float64)
    yd = y.astype(np.float64)
    exact = 0.5 * yd * (1.0 + erf(yd / np.sqrt(2.0)))
    # the tanh form is within 5e-4 of the erf GELU; the bf16 rounding adds half an ulp
    assert np.all(np.abs(g - exact) <= 5e-4 + 2.0 ** -8 * np.abs(exact))


def test_f64_to_bf16_agrees_with_float32_path_on_float32_values():
    rng = np.random.default_rng(0)
    b = rng.integers(0, 2 ** 32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    f = b.view(np.float32)
    f = f[np.isfinite(f)]
    np.testing.assert_array_equal(orc.f64_to_bf16_bits(f.astype(np.float64)), orc.f32_to_bf16_bits(f))


def test_f64_to_bf16_single_rounding():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7; a float64 bit either side decides
    x = np.array([1 + 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -8 - 2.0 ** -40,
                  1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8 + 2.0 ** -40),
                  # below 2^-126: quantum 2^-133; 2.5 quanta ties to 2, a hair more goes to 3
                  2.5 * 2.0 ** -133, 2.5 * 2.0 ** -133 * (1 + 2.0 ** -40), 0.5 * 2.0 ** -133,
                  0.5 * 2.0 ** -133 * (1 + 2.0 ** -40), -0.0, 3.4e38, -1e300])
    want = [0x3F80, 0x3F81, 0x3F80, 0x3F82, 0xBF81, 0x0002, 0x0003, 0x0000, 0x0001, 0x8000,
            0x7F80, 0xFF80]
    np.testing.assert_array_equal(orc.f64_to_bf16_bits(x), np.array(want, np.uint16))
    # a float32 detour would round twice: 1 + 2^-8 + 2^-30 becomes the tie 1 + 2^-8 in float32
    assert orc.f32_to_bf16_bits(np.array([1 + 2.0 ** -8 + 2.0 ** -30], np.float32))[0] == 0x3F80
    assert orc.f64_to_bf16_bits(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81


def test_gelu_special_values():
    y = np.array([0.0, -0.0, 1.0, -1.0, 16.0, 123.5, -16.0, -0.5], np.float32)
    g = orc.gelu_bf16(y)
    assert g[0] == 0.0 and not np.signbit(g[0])
    assert g[1] == 0.0 and np.signbit(g[1])
    # gelu(1) = 0.841192 -> 215/256; gelu(-1) = -0.158808 -> -163/1024
    assert g[2] == 0.83984375 and g[3] == -0.1591796875
    assert g[4] == 16.0 and g[5] == 123.5               # 1 - gelu(y)/y far below half an ulp
    assert g[6] == 0.0 and np.signbit(g[6])             # |gelu(-16)| ~ 1e-137: a negative zero
    assert g[7] == -0.154296875                         # gelu(-0.5) = -0.154286


def test_ffn_hidden_is_bf16():
    y = np.linspace(-8, 8, 1001).astype(np.float32)
    h = orc.ffn_hidden(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(y)))
    np.testing.assert_array_equal(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(h)), h)
