"""Pins of the oracle's float32 GELU (the FFN activation between the two
projections): exp against float64 exp, GELU against the float64 closed form
0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), special values."""
import numpy as np

from oracle import w4a4_oracle as orc


def test_exp_within_two_ulp_of_float64():
    z = np.linspace(-87.0, 88.0, 1_000_001).astype(np.float32)
    e = orc.exp_f32(z).astype(np.float64)
    ref = np.exp(z.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(e - ref) / ulp) <= 2.0
    # exactly representable points
    assert orc.exp_f32(np.array([0.0], np.float32))[0] == 1.0


def test_gelu_matches_closed_form():
    x = np.linspace(-20.0, 20.0, 2_000_001).astype(np.float32)
    g = orc.gelu_f32(x).astype(np.float64)
    xd = x.astype(np.float64)
    ref = 0.5 * xd * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)))
    big = np.abs(ref) > 1e-2
    assert np.max(np.abs(g - ref)[big] / np.abs(ref[big])) < 1e-6
    assert np.max(np.abs(g - ref)) < 1e-6


def test_gelu_special_values():
    x = np.array([0.0, -0.0, 10.0, 123.5, -12.0, 1.0, -1.0], np.float32)
    g = orc.gelu_f32(x)
    assert g[0] == 0.0 and not np.signbit(g[0])
    assert g[1] == 0.0 and np.signbit(g[1])
    assert g[2] == 10.0 and g[3] == 123.5              # exp term below half an ulp of 1
    assert -1e-30 < g[4] < 0.0
    np.testing.assert_allclose(g[5:], [0.8411920071, -0.1588079929], rtol=1e-6)


def test_ffn_hidden_is_bf16():
    y = np.linspace(-8, 8, 1001).astype(np.float32)
    h = orc.ffn_hidden(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(y)))
    np.testing.assert_array_equal(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(h)), h)
