"""Pins for the oracle's whole path (no GPU).

Each test fixes the oracle against something other than itself: the FP64
fold identity of the SmoothQuant section, the special cases the method
reduces to (k = 0 is a plain MXFP4 GEMM, k = d_in a bfloat16 GEMM, s = 1
leaves X untouched), a brute-force check of the top-k definition, the
monotonicity of rounding that lets the score be read from act_scale, and
error bounds against the unquantised product.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import w4a4_oracle as orc


def _bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy()


def _small(T=64, d_in=96, d_out=48, seed=0, n_out=4):
    spec = synth.XSpec("student3", 0.3, n_out, 8.0, 30.0)
    X = _bf16_np(synth.gen_x(spec, T, d_in, seed))
    W = _bf16_np(synth.gen_w(synth.WSpec(0.02), d_out, d_in, seed + 1))
    return X, W


@pytest.mark.parametrize("alpha", [0.5, 0.7])
def test_fold_identity_fp64(alpha):
    """(X ⊘ s)(s ⊙ W) = XW in exact arithmetic (W4A4 review §3.2, fold equation)."""
    X, W = _small()
    act = orc.col_absmax(X)
    wsc = orc.col_absmax(W)
    s32, _ = orc.smoothing_factors(act, wsc, alpha)
    s = s32.astype(np.float64)
    lhs = orc.smooth_activation(X.astype(np.float64), 1.0 / s) @ orc.fold_weight(W.astype(np.float64), s).T
    rhs = X.astype(np.float64) @ W.astype(np.float64).T
    rel = np.abs(lhs - rhs).max() / np.abs(rhs).max()
    assert rel <= 1e-12


def test_fold_axis_matters():
    X, W = _small(d_in=64, d_out=64)
    s, inv_s = orc.smoothing_factors(orc.col_absmax(X), orc.col_absmax(W), 0.5)
    s = s.astype(np.float64)
    good = orc.smooth_activation(X.astype(np.float64), 1 / s) @ orc.fold_weight(W.astype(np.float64), s).T
    wrong = orc.smooth_activation(X.astype(np.float64), 1 / s) @ (W.astype(np.float64) * s[:, None]).T
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.abs(good - ref).max() < 1e-9 * np.abs(ref).max()
    assert np.abs(wrong - ref).max() > 1e-3 * np.abs(ref).max()


def test_smoothing_closed_forms():
    # alpha = 0.5, a = 16, w = 1 -> s = 4 ; a = 1, w = 0.25 -> s = 1 / 0.5 = 2
    s, inv_s = orc.smoothing_factors(np.array([16.0, 1.0], np.float32),
                                     np.array([1.0, 0.25], np.float32), 0.5)
    np.testing.assert_array_equal(s, [4.0, 2.0])
    np.testing.assert_array_equal(inv_s, [0.25, 0.5])
    # alpha = 0.7, a = 2^10, w = 2^-10 -> s = 2^7 * 2^3 = 2^10
    s, _ = orc.smoothing_factors(np.array([1024.0], np.float32), np.array([2.0**-10], np.float32), 0.7)
    assert abs(float(s[0]) - 1024.0) <= 1024.0 * 2**-22
    # the activation magnitude carries exponent alpha, the weight's 1 - alpha
    # (review sec. 3.2, eq. s_j): alpha = 0.7, a = 2^10, w = 1 -> s = 2^7;
    # a = 1, w = 2^10 -> s = 2^-3 (exchanged exponents would give 2^3, 2^-7)
    s, _ = orc.smoothing_factors(np.array([1024.0, 1.0], np.float32),
                                 np.array([1.0, 1024.0], np.float32), 0.7)
    np.testing.assert_allclose(s.astype(np.float64), [128.0, 0.125], rtol=2**-22)
    # zero magnitudes are clamped at 1e-5: a = 0, w = 0, alpha = 0.5 -> s = 1e-5^0.5 / 1e-5^0.5 = 1
    s, _ = orc.smoothing_factors(np.zeros(1, np.float32), np.zeros(1, np.float32), 0.5)
    assert s[0] == 1.0


def test_smoothing_balances_ranges_at_half():
    """At alpha = 0.5 the smoothed activation channel max equals the folded
    weight channel max (both are sqrt(a_j w_j)), the balance SmoothQuant targets."""
    X, W = _small(T=128, d_in=64, d_out=64)
    act, wsc = orc.col_absmax(X), orc.col_absmax(W)
    s, inv_s = orc.smoothing_factors(act, wsc, 0.5)
    xs = orc.col_absmax(orc.smooth_activation(X.astype(np.float64), 1.0 / s.astype(np.float64)))
    ws = orc.col_absmax(orc.fold_weight(W.astype(np.float64), s.astype(np.float64)))
    np.testing.assert_allclose(xs, ws, rtol=1e-6)
    np.testing.assert_allclose(xs, np.sqrt(act.astype(np.float64) * wsc), rtol=1e-6)


def test_calibration_over_batches_equals_their_concatenation():
    """Calibrating on several batches is calibrating on their union: each
    per-channel magnitude is a max over every calibration token (review
    sec. 3.2, magnitudes collected over the calibration data, which the
    pipeline gathers in batches across timesteps)."""
    X, W = _small(T=192, d_in=96, n_out=0)
    X1, X2, X3 = X[:64].copy(), X[64:128].copy(), X[128:].copy()
    X2[:, 5] *= 64.0           # an outlier channel seen only in the second batch
    X3[:, 70] *= 128.0         # and one seen only in the third (powers of 2: exact)
    full = orc.calibrate(np.vstack([X1, X2, X3]), W, 0.6, 4)
    parts = orc.calibrate([X1, X2, X3], W, 0.6, 4)
    for key in ("act_scale", "w_scale", "s", "inv_s", "score", "O", "J"):
        np.testing.assert_array_equal(parts[key], full[key], err_msg=key)
    assert {5, 70} <= set(full["O"].tolist())


def test_smoothing_product_is_one_float32_multiply():
    """x * inv_s is rounded to float32 before it is encoded (the reading of
    review sec. 3.2's "divide by s": one IEEE float32 multiply by fl32(1/s)).
    Hand-worked: x = 0.25390625 (bf16), inv_s = 0.98461538553237915 (float32);
    the exact product is 0.25 + 2.3e-10, its float32 rounding exactly 0.25.
    With 4.0 in the same block (scale 2^0), 0.25 is the tie between the E2M1
    codes for 0 and 0.5 and goes to the even one, 0; the unrounded product
    would encode as 0.5."""
    x = np.float32(0.25390625)
    inv = np.float32(0.98461538553237915)
    assert np.float32(x * inv) == np.float32(0.25)
    assert float(x) * float(inv) > 0.25
    X = np.zeros((1, 32), np.float32)
    X[0, 0], X[0, 1] = x, 4.0
    inv_s = np.ones(32, np.float32)
    inv_s[0] = inv
    out = orc.prep_activation(X, inv_s, np.zeros(0, np.int32), np.arange(32, dtype=np.int32))
    assert out["sfa"][0, 0] == 127                      # shared exponent 0
    assert out["aq"][0, 0] == 0x60                      # codes 0 (x) and 6 (4.0)


def test_score_equals_scaled_act_scale():
    """max_t fl32(|x| * inv_s) = fl32(max_t |x| * inv_s): rounding is monotone,
    so the score needs no second pass over X."""
    X, W = _small(T=300, d_in=160)
    act = orc.col_absmax(X)
    _, inv_s = orc.smoothing_factors(act, orc.col_absmax(W), 0.6)
    direct = orc.outlier_scores(X, inv_s)
    shortcut = (act * inv_s).astype(np.float32)
    np.testing.assert_array_equal(direct, shortcut)


def test_topk_definition_brute_force():
    rng = np.random.default_rng(1)
    for trial in range(40):
        d = int(rng.integers(1, 40))
        score = rng.integers(0, 6, d).astype(np.float32)   # many ties on purpose
        k = int(rng.integers(0, d + 1))
        O, J = orc.select_outliers(score, k)
        assert len(O) == k and len(J) == d - k
        assert np.all(np.diff(O) > 0) and np.all(np.diff(J) > 0)
        assert sorted(np.concatenate([O, J]).tolist()) == list(range(d))
        for j in O:
            for i in J:
                assert score[j] > score[i] or (score[j] == score[i] and j < i)


def test_topk_edges():
    sc = np.array([1, 3, 3, 2], np.float32)
    O, J = orc.select_outliers(sc, 0)
    assert O.size == 0 and J.tolist() == [0, 1, 2, 3]
    O, J = orc.select_outliers(sc, 1)
    assert O.tolist() == [1] and J.tolist() == [0, 2, 3]
    O, J = orc.select_outliers(sc, 4)
    assert O.tolist() == [0, 1, 2, 3] and J.size == 0
    with pytest.raises(ValueError):
        orc.select_outliers(sc, 5)


def test_identity_smoothing_is_plain_mxfp4():
    """s = 1: prep quantises X itself; the O columns are copied unchanged."""
    X, _ = _small(T=40, d_in=80)
    O = np.array([3, 17, 40], np.int32)
    J = np.setdiff1d(np.arange(80), O).astype(np.int32)
    pa = orc.prep_activation(X, np.ones(80, np.float32), O, J)
    np.testing.assert_array_equal(orc.bf16_bits_to_f32(pa["xo"]), X[:, O])
    nb = orc.n_blocks(len(J))
    XJ = np.zeros((40, nb * 32), np.float32)
    XJ[:, :len(J)] = X[:, J]
    sc, codes = orc.mxfp4_quantize_blocks(XJ.reshape(40, nb, 32))
    np.testing.assert_array_equal(pa["sfa"], sc)
    np.testing.assert_array_equal(pa["aq"], orc.pack_nibbles(codes.reshape(40, -1)))


def test_k0_is_plain_mx_gemm_and_bounded():
    """k = 0: the second branch vanishes; Y is the FP64 product of the
    dequantised operands, and it stays within the element-wise quantisation
    error bound of XW."""
    X, W = _small(T=32, d_in=64, d_out=16)
    Y, p = orc.linear_reference(X, W, 0.5, 0)
    assert p["xo"].shape[1] == 0 and p["w_hp"].shape[1] == 0
    A = orc.dequant_mxfp4(p["aq"], p["sfa"])
    B = orc.dequant_mxfp4(p["wq"], p["sfb"])
    np.testing.assert_array_equal(Y, A @ B.T)
    # bound from the quantiser definition: |deq(v) - v| <= 2^e * (half spacing or saturation)
    Vx = orc.smooth_activation(X.astype(np.float32), p["inv_s"]).astype(np.float64)
    Vw = orc.fold_weight(W.astype(np.float32), p["s"]).astype(np.float64)

    def err_bound(V, sf):
        e = np.repeat(sf.astype(np.float64) - 127, 32, axis=1)[:, :V.shape[1]]
        q = np.abs(V) * 2.0 ** -e
        half = np.where(q < 2, 0.25, np.where(q < 4, 0.5, np.where(q <= 6, 1.0, q - 6)))
        return half * 2.0 ** e

    ex, ew = err_bound(Vx, p["sfa"]), err_bound(Vw, p["sfb"])
    bound = (ex @ np.abs(Vw).T + np.abs(Vx) @ ew.T + ex @ ew.T) * (1 + 1e-6)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    # Vx Vw^T differs from XW only by the fl32 roundings of the smoothing (2^-23 relative)
    slack = 4 * 2.0**-23 * (np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T)
    assert np.all(np.abs(Y - exact) <= bound + slack)


def test_k_equals_din_is_bf16_gemm():
    """k = d_in: no column is quantised; Y is the product of the bf16-rounded
    smoothed operands and stays within bf16 rounding of XW."""
    X, W = _small(T=24, d_in=48, d_out=20)
    Y, p = orc.linear_reference(X, W, 0.7, 48)
    assert p["aq"].shape[1] == 0 and p["xo"].shape[1] == 48
    XO = orc.bf16_bits_to_f32(p["xo"]).astype(np.float64)
    WO = orc.bf16_bits_to_f32(p["w_hp"]).astype(np.float64)
    np.testing.assert_array_equal(Y, XO @ WO.T)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    mag = np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T
    # each operand: bf16 rounding (unit roundoff 2^-8: 8 significant bits)
    # plus the fl32 roundings of the product and of inv_s
    eps = 2.0**-8 + 2 * 2.0**-23
    assert np.all(np.abs(Y - exact) <= (2 * eps + eps * eps) * mag * (1 + 1e-9))


def test_split_sum_recombines():
    """Y = X_J W_J + X_O W_O: with quantisation replaced by the identity the two
    branches add up to the full product.  Checked by brute force: the oracle's
    O/J split of columns, the compaction and the gathered bf16 columns index the
    same channels on both operands."""
    X, W = _small(T=16, d_in=70, d_out=12)
    Y, p = orc.linear_reference(X, W, 0.5, 9)
    O, J = p["O"], p["J"]
    XO = orc.bf16_bits_to_f32(p["xo"]).astype(np.float64)
    WO = orc.bf16_bits_to_f32(p["w_hp"]).astype(np.float64)
    Vx = orc.smooth_activation(X.astype(np.float32), p["inv_s"])
    Vw = orc.fold_weight(W.astype(np.float32), p["s"])
    for t in range(4):
        for n in range(4):
            o_branch = sum(float(XO[t, i]) * float(WO[n, i]) for i in range(len(O)))
            o_direct = sum(float(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(Vx[t, j:j + 1]))[0]) *
                           float(orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(Vw[n, j:j + 1]))[0])
                           for j in O)
            assert abs(o_branch - o_direct) <= 1e-12 * (1 + abs(o_direct))
    A = orc.dequant_mxfp4(p["aq"], p["sfa"])
    B = orc.dequant_mxfp4(p["wq"], p["sfb"])
    j_branch = A @ B.T
    np.testing.assert_allclose(Y, j_branch + XO @ WO.T, rtol=0, atol=1e-12)
    # the J-branch, compacted, covers exactly the J channels: dequantised values
    # stay within the quantisation error of the smoothed J columns
    assert np.all(np.abs(A[:, :len(J)] - Vx[:, J]) <= np.abs(Vx[:, J]).max() * 0.5 + 1e-30)


def test_32x32_tiles_share_one_scale():
    X, W = _small(T=8, d_in=256, d_out=80)
    _, p = orc.linear_reference(X, W, 0.5, 5, layout=orc.LAYOUT_32x32)
    sfb = p["sfb"]
    for g in range(0, 80, 32):
        tile = sfb[g:g + 32]
        assert np.all(tile == tile[0:1])
    # the tile scale is the one of the tile's largest element
    Vw = orc.fold_weight(W.astype(np.float32), p["s"])[:, p["J"]]
    nb = sfb.shape[1]
    VJ = np.zeros((80, nb * 32), np.float32)
    VJ[:, :Vw.shape[1]] = Vw
    amax = np.abs(VJ[0:32, 0:32]).max()
    assert int(sfb[0, 0]) == int(orc.mx_shared_exponent(np.array([amax]))[0]) + 127


def _pack_plain(W, layout):
    """pack_weight with s = 1, no outliers: plain per-row encoding of W."""
    d_in = W.shape[1]
    return orc.pack_weight(W.astype(np.float32), np.ones(d_in, np.float32),
                           np.zeros(0, np.int64), np.arange(d_in), layout)


def test_128x1_stripe_hand_worked():
    """[review §3.4] 128x1 K-major stripe: 4 consecutive MX blocks of a row
    share the exponent of the stripe's largest element (values worked by hand
    on the E2M1 grid)."""
    W = np.zeros((1, 256), np.float32)
    W[0, 0] = 6.0                                        # stripe 0 amax 6 -> e = 0
    W[0, 32:37] = [0.25, 0.75, -2.5, 0.09375, 1.5]       # block 1, coded with e = 0
    W[0, 160] = 0.09375                                  # stripe 1 amax 3/32 -> e = -6
    p = _pack_plain(W, orc.LAYOUT_128x1)
    assert p["sfb"][0].tolist() == [127] * 4 + [121] * 4
    codes = orc.unpack_nibbles(p["wq"])[0]
    assert codes[0] == 0x7                               # 6
    assert codes[32:37].tolist() == [0x0, 0x2, 0xC, 0x0, 0x3]   # 0.25->0 (tie), 0.75->1, -2.5->-2 (tie), 3/32->0, 1.5
    assert codes[160] == 0x7                             # 3/32 * 64 = 6
    # the 32x1 layout gives block 1 its own exponent: amax 2.5 -> e = -1
    q = _pack_plain(W, orc.LAYOUT_32x1)
    assert q["sfb"][0, 1] == 126 and q["sfb"][0, 0] == 127 and q["sfb"][0, 5] == 121


def test_128x1_equals_32x1_when_blocks_share_amax():
    """If the 4 blocks of every stripe have the same amax, sharing it changes
    nothing: the 128x1 packing equals the 32x1 packing."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((40, 512)) * 0.3).astype(np.float32)
    W = np.clip(W, -1.0, 1.0)
    W[:, ::32] = 1.5 * np.sign(W[:, ::32] + 0.5)         # every block holds +-1.5 as its max
    a = _pack_plain(W, orc.LAYOUT_128x1)
    b = _pack_plain(W, orc.LAYOUT_32x1)
    np.testing.assert_array_equal(a["sfb"], b["sfb"])
    np.testing.assert_array_equal(a["wq"], b["wq"])


def test_128x1_stripes_share_scale_and_saturate_at_max():
    X, W = _small(T=8, d_in=600, d_out=48)
    _, p = orc.linear_reference(X, W, 0.6, 7, layout=orc.LAYOUT_128x1)
    sfb = p["sfb"]
    nb = sfb.shape[1]
    for b0 in range(0, nb, 4):
        st = sfb[:, b0:b0 + 4]
        assert np.all(st == st[:, 0:1])
    # the stripe maximum codes to magnitude 6 or 7 (|q| in [4, 8))
    codes = orc.unpack_nibbles(p["wq"]) & 0x7
    Vw = orc.fold_weight(W.astype(np.float32), p["s"])[:, p["J"]]
    for r in range(48):
        for b0 in range(0, nb, 4):
            seg = np.abs(Vw[r, b0 * 32:(b0 + 4) * 32])
            if seg.size and seg.max() > 0:
                i = b0 * 32 + int(np.argmax(seg))
                assert codes[r, i] in (6, 7)


def test_search_layer_prefers_protecting_planted_outliers():
    """On the tiny workload (8 planted heavy channels), keeping them in bf16
    (k = 8) beats k = 0 at every alpha, all-bf16 (k = d_in) is near exact,
    and the returned best is the table's minimum."""
    L = synth.TINY
    Xt, Wt = synth.gen_layer(L, "cpu")
    X, W = Xt.float().numpy()[:64], Wt.float().numpy()
    best, err = orc.search_layer(X, W, alphas=(0.3, 0.5, 0.7), ks=(0, 8, L.d_in))
    for a in (0.3, 0.5, 0.7):
        assert err[(a, 8, 0)] < 0.8 * err[(a, 0, 0)]
        assert err[(a, L.d_in, 0)] < 5e-3          # bf16 rounding of smoothed operands only
    assert best == min(err, key=lambda c: (err[c], c[1]))
    assert best[1] == L.d_in


def test_tiny_generator_matches_pages_statistics():
    """The tiny workload's planted channels exceed 6.0, weights stay below 0.6
    (review §3.1), and after smoothing the planted channels are the top-8."""
    L = synth.TINY
    X, W = synth.gen_layer(L)
    X, W = _bf16_np(X), _bf16_np(W)
    planted = synth.outlier_columns(L.x, L.d_in, L.seed).numpy()
    act = orc.col_absmax(X)
    assert np.all(act[planted] > 6.0)
    assert orc.col_absmax(W).max() < 0.6
    c = orc.calibrate(X, W, L.alpha, L.k)
    assert sorted(c["O"].tolist()) == sorted(planted.tolist())


def test_smoothing_and_splitting_help():
    """Qualitative ordering stated in review §3.5: smoothing + splitting gives
    a better SNR than plain W4A4 rounding on heavy-tailed activations."""
    spec = synth.XSpec("student3", 0.3, 8, 8.0, 30.0)
    X = _bf16_np(synth.gen_x(spec, 256, 512, 0))
    W = _bf16_np(synth.gen_w(synth.WSpec(0.02), 128, 512, 1))
    exact = X.astype(np.float64) @ W.astype(np.float64).T

    def snr(Y):
        return 10 * np.log10((exact**2).sum() / ((Y - exact)**2).sum())

    O0 = np.zeros(0, np.int32)
    J0 = np.arange(512, dtype=np.int32)
    s1 = np.ones(512, np.float32)
    pw = orc.pack_weight(W, s1, O0, J0)
    pa = orc.prep_activation(X, s1, O0, J0)
    plain = orc.dual_branch_product(pa["aq"], pa["sfa"], pa["xo"], pw["wq"], pw["sfb"], pw["w_hp"])
    ours, _ = orc.linear_reference(X, W, 0.5, 8)
    assert snr(ours) > snr(plain)


def test_non_finite_activations_hand_worked():
    # Where the pages say nothing, IEEE float32 arithmetic and the E8M0 codes
    # decide (see the oracle's readings).  d_in = 64, O = {0, 1}: X_O holds
    # columns 0 and 1; J = 2 .. 63 forms block 0 (columns 2 .. 33) and block 1
    # (34 .. 63 and two zeros).  Values worked by hand:
    #  row 0: x00 = 2^127 times inv_s 4 overflows -> +inf -> bf16 0x7F80;
    #         x01 = NaN -> 0x7FC0; x02 = -inf -> block 0 amax inf, e = 127
    #         (code 254), code 0xF; x03 = 1.5 2^126 -> q = 0.75 -> code 2;
    #         x04 = 1 -> q = 2^-127 -> code 0; x34 = NaN -> block 1 code 255,
    #         all codes 0.
    #  row 1: x05 = 2^127 times inv_s 2 -> 2^128 overflows -> +inf: block 0
    #         code 254, its code (position 3) 7; x06 = -2^126 -> q = -0.5 ->
    #         code 9; x01 = -NaN (sign set) -> still 0x7FC0; block 1 all zero
    #         -> code 0.
    d_in = 64
    O = np.array([0, 1], np.int32)
    J = np.arange(2, d_in, dtype=np.int32)
    inv_s = np.ones(d_in, np.float32)
    inv_s[0] = 4.0
    inv_s[5] = 2.0
    X = np.zeros((2, d_in), np.float32)
    X[0, [0, 1, 2, 3, 4, 34]] = [2.0 ** 127, np.nan, -np.inf, 1.5 * 2.0 ** 126, 1.0, np.nan]
    X[1, [1, 5, 6]] = [-np.nan, 2.0 ** 127, -2.0 ** 126]
    out = orc.prep_activation(X, inv_s, O, J)
    assert out["xo"][0].tolist() == [0x7F80, 0x7FC0]
    assert out["xo"][1].tolist() == [0x0000, 0x7FC0]
    assert out["sfa"].tolist() == [[254, 255], [254, 0]]
    codes = orc.unpack_nibbles(out["aq"])
    assert codes[0, :3].tolist() == [0xF, 0x2, 0x0] and not codes[0, 3:].any()
    assert codes[1, :5].tolist() == [0, 0, 0, 0x7, 0x9] and not codes[1, 5:].any()


def test_calibration_refuses_non_finite_magnitudes():
    # s_j = a^alpha / w^(1 - alpha) has no value for an infinite or NaN magnitude
    a = np.ones(8, np.float32)
    w = np.ones(8, np.float32)
    for bad in (np.inf, np.nan):
        for which in ("act", "w"):
            aa, ww = a.copy(), w.copy()
            (aa if which == "act" else ww)[3] = bad
            with pytest.raises(ValueError):
                orc.smoothing_factors(aa, ww, 0.5)
    s, inv_s = orc.smoothing_factors(a, w, 0.5)
    assert (s == 1).all() and (inv_s == 1).all()


def test_search_layer_hand_worked():
    """The relative Frobenius metric and the tie rule on a case whose every
    candidate was worked by hand (tests/golden/search_layer_hand.txt)."""
    from tests import search_hand_case as hc
    X, W = hc.inputs()
    table, best_hand = hc.expected()
    best, err = orc.search_layer(X, W, hc.ALPHAS, hc.KS)
    assert set(err) == set(table)
    for c, e in table.items():
        assert abs(err[c] - e) <= 1e-12, (c, err[c], e)
    assert best == best_hand


def test_ffn_chain_interval_contains_every_up_output_in_the_band():
    """The interval the FFN chain test uses (tests/ffn_bounds.py) contains the
    oracle's own down product for up-layer outputs drawn anywhere in the
    band: the bound is sound (it is not a reading of the pages, it is how the
    GPU test compares an end-to-end result with an oracle chain from X)."""
    from tests import ffn_bounds as fb
    rng = np.random.default_rng(0)
    T, dm, dff = 24, 64, 160
    q = lambda a: orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(a.astype(np.float32)))
    X = q(rng.standard_t(3, (T, dm)) * 0.3)
    Wu, Wd = q(rng.normal(size=(dff, dm)) * 0.05), q(rng.normal(size=(dm, dff)) * 0.05)
    cu = orc.calibrate(X, Wu, 0.6, 4)
    wu = orc.pack_weight(Wu, cu["s"], cu["O"], cu["J"])
    au = orc.prep_activation(X, cu["inv_s"], cu["O"], cu["J"])
    Yu = orc.dual_branch_product(au["aq"], au["sfa"], au["xo"], wu["wq"], wu["sfb"], wu["w_hp"])
    cd = orc.calibrate(orc.ffn_hidden(q(Yu)), Wd, 0.7, 6)
    tol = fb.up_tolerance(Yu)
    ylo, yhi = fb.bf16_round_out(Yu - tol, Yu + tol)
    assert (ylo <= Yu - tol).all() and (yhi >= Yu + tol).all()
    Ylo, Yhi = fb.down_interval(Yu, tol, cd, Wd, orc.LAYOUT_32x1)
    wd = orc.pack_weight(Wd, cd["s"], cd["O"], cd["J"])
    for _ in range(8):
        yb = np.clip(q(Yu + tol * rng.uniform(-1, 1, Yu.shape)), ylo, yhi)
        ad = orc.prep_activation(orc.ffn_hidden(yb), cd["inv_s"], cd["O"], cd["J"])
        Yd = orc.dual_branch_product(ad["aq"], ad["sfa"], ad["xo"], wd["wq"], wd["sfb"], wd["w_hp"])
        assert (Yd >= Ylo - 1e-9).all() and (Yd <= Yhi + 1e-9).all()
    # and a chain that leaves the band (GELU skipped) falls outside somewhere
    ad = orc.prep_activation(q(Yu), cd["inv_s"], cd["O"], cd["J"])
    Yd = orc.dual_branch_product(ad["aq"], ad["sfa"], ad["xo"], wd["wq"], wd["sfb"], wd["w_hp"])
    assert ((Yd < Ylo - 1e-9) | (Yd > Yhi + 1e-9)).any()
