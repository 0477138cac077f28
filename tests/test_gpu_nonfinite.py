"""Non-finite values on the GPU against the oracle's reading of them.

The pages say nothing about inf or NaN; the oracle reads them by IEEE float32
arithmetic and the E8M0 encoding (a block holding a NaN gets scale code 0xFF
and zero element codes; a block holding an infinity gets e = 127, its
infinities saturate to +-6; a NaN in the bf16 branch is written 0x7FC0).
Every activation and weight encoder of the library must give the same bits
on every bf16 pattern, infinities and NaNs included, and on products that
overflow float32.  Calibration magnitudes that are not finite are reported
through the device error word.
"""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from w4a4_mxfp4_outlier_b200 import ffn
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu
from tests.test_gpu_parity import _compare_prep, _manual_pw

pytestmark = pytest.mark.gpu

ALL_BITS = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def _rows_of(vals, d_in):
    T = -(-vals.size // d_in)
    Xb = np.zeros(T * d_in, np.uint16)
    Xb[:vals.size] = vals
    return Xb.reshape(T, d_in)


# every bf16 pattern (inf and NaN among them) through both prep kernels: the
# block-per-lane form (d_in 512) and the 8-columns-per-lane form (d_in 16384);
# "overflow": inv_s up to 2^90, so large finite x give products beyond float32
@pytest.mark.parametrize("d_in", [512, 16384])
@pytest.mark.parametrize("variant", ["identity", "shuffled", "random_inv_s", "overflow"])
def test_prep_encodes_every_bf16_pattern(variant, d_in):
    rng = np.random.default_rng(1)
    vals = ALL_BITS if variant == "identity" else rng.permutation(ALL_BITS)
    Xb = _rows_of(vals, d_in)
    T = Xb.shape[0]
    inv_s = np.ones(d_in, np.float32)
    if variant == "random_inv_s":
        inv_s = rng.uniform(0.01, 4.0, d_in).astype(np.float32)
    elif variant == "overflow":
        inv_s = np.exp2(rng.uniform(0.0, 90.0, d_in)).astype(np.float32)
    O = (np.sort(rng.choice(d_in, 7, replace=False)).astype(np.int32)
         if variant != "identity" else np.zeros(0, np.int32))
    J = np.setdiff1d(np.arange(d_in), O).astype(np.int32)
    pw = _manual_pw(d_in, len(O), inv_s, O, J)
    X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
    act = w4.alloc_act(T, pw)
    w4.prep_act(X, pw, act)
    torch.cuda.synchronize()
    ref = orc.prep_activation(orc.bf16_bits_to_f32(Xb), inv_s, O, J)
    assert (ref["sfa"] == 255).any()                          # NaN blocks occur
    if variant != "identity":                                  # (in order, every inf sits by a NaN)
        assert (ref["sfa"] == 254).any()                       # and blocks with an infinity
    _compare_prep(ref, act, pw, T)


# every bf16 pattern as weights, packed in all three scale layouts (32x1 and
# 128x1 stream through the prep kernel, 32x32 tiles through their own kernel)
@pytest.mark.parametrize("layout", [0, 1, 2])
def test_pack_encodes_every_bf16_pattern(layout):
    rng = np.random.default_rng(3)
    d_in, d_out, k = 512, 128, 5
    vals = rng.permutation(ALL_BITS)
    Wb = vals[:d_out * d_in].reshape(d_out, d_in)
    s = np.exp2(rng.uniform(-4.0, 60.0, d_in)).astype(np.float32)
    O = np.sort(rng.choice(d_in, k, replace=False)).astype(np.int32)
    J = np.setdiff1d(np.arange(d_in), O).astype(np.int32)
    pw = w4.alloc_packed(d_in, d_out, k, layout)
    pw.s.copy_(torch.from_numpy(s))
    pw.inv_s.copy_(torch.from_numpy((1.0 / s.astype(np.float64)).astype(np.float32)))
    pw.O.copy_(torch.from_numpy(O))
    pw.jmap.copy_(torch.from_numpy(J))
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    w4.pack_weight(W, pw)
    torch.cuda.synchronize()
    ref = orc.pack_weight(orc.bf16_bits_to_f32(Wb), s, O, J, layout)
    assert (ref["sfb"] == 255).any() and (ref["sfb"] == 254).any()
    d = pw.dims
    nb = ref["sfb"].shape[1]
    np.testing.assert_array_equal(pw.wq.view(d_out, -1).cpu().numpy()[:, :nb * 16], ref["wq"])
    sfb = gu.sf_canonical(pw.sfb, d.sfb_rows, d.nblk, nb)
    np.testing.assert_array_equal(sfb[:d_out, :nb], ref["sfb"])
    np.testing.assert_array_equal(gu.bf16_bits(pw.w_hp).reshape(d_out, -1)[:, :k], ref["w_hp"])


def test_calibration_reports_non_finite_magnitudes():
    L = synth.TINY
    X, W = gu.gen(L)
    w4.last_error(clear=True)
    pw = w4.calibrate(X, W, L.alpha, L.k)
    assert w4.last_error()[0] == w4.OK
    for bad in (float("inf"), float("nan")):
        Xb = X.clone()
        Xb[17, 100] = bad
        w4.calibrate(Xb, W, L.alpha, L.k)
        st, bits = w4.last_error(clear=True)
        assert st == w4.ERR_NONFINITE_CALIB, (bad, hex(bits))
        assert w4.last_error()[0] == w4.OK          # cleared
    Wb = W.clone()
    Wb[3, 7] = float("-inf")
    w4.calibrate(X, Wb, L.alpha, L.k)
    assert w4.last_error(clear=True)[0] == w4.ERR_NONFINITE_CALIB


def _oracle_y(X, W, pw, layout):
    c = gu.oracle_calib_from_gpu(pw)
    rw = orc.pack_weight(gu.to_np_f32(W), c["s"], c["O"], c["J"], layout)
    ra = orc.prep_activation(gu.to_np_f32(X), c["inv_s"], c["O"], c["J"])
    with np.errstate(invalid="ignore", over="ignore"):
        return orc.dual_branch_product(ra["aq"], ra["sfa"], ra["xo"], rw["wq"], rw["sfb"],
                                       rw["w_hp"]), c


@pytest.mark.parametrize("T", [100, 300])                 # single-CTA and pair GEMM
def test_linear_rows_with_nan_inputs_are_nan(T):
    """Calibrated on finite data, run on rows that hold a NaN (in a 4-bit
    column or an outlier column): such a row's Y is NaN in every output, on
    both sides (E8M0 0xFF, or a NaN in the bf16 branch, reaches every column);
    every other row is within the usual tolerance."""
    L = synth.Layer("nonfinite", T, 512, 384, 0.6, 8, 0, synth.X_UP, synth.W_UP, seed=21)
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k)
    torch.cuda.synchronize()
    O = pw.O.cpu().numpy()
    J = pw.jmap.cpu().numpy()
    Xd = X.clone()
    Xd[3, int(J[40])] = float("nan")
    Xd[7, int(O[2])] = float("nan")
    Xd[T - 1, int(J[0])] = float("-nan")
    ws = torch.empty(w4.workspace_size(T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Y = torch.empty((T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(Xd, pw, ws, Y)
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)
    Y_ref, _ = _oracle_y(Xd, W, pw, 0)
    Yg = gu.to_np_f32(Y).astype(np.float64)
    nan_rows = [3, 7, T - 1]
    assert np.isnan(Y_ref[nan_rows]).all()
    assert np.isnan(Yg[nan_rows]).all()
    ok = np.setdiff1d(np.arange(T), nan_rows)
    gu.check_tolerance(Yg[ok], Y_ref[ok], "finite rows")


def test_fused_ffn_epilogue_on_non_finite_rows():
    """NaN and infinite up-layer outputs through the fused epilogue: the down
    layer's operands equal the oracle's prep of bf16(gelu(Y_up)) bit for bit
    (GELU of +inf is +inf, of -inf and NaN a NaN; then the encoding rules)."""
    T, d_model, d_ff = 300, 512, 1376
    Lx = synth.Layer("ffn_up_nf", T, d_model, d_ff, 0.6, 8, 0,
                     synth.XSpec("student3", 0.3, 6, 8.0, 30.0), synth.WSpec(0.02), seed=7)
    X, W_up = gu.gen(Lx)
    W_down = synth.gen_w(synth.WSpec(0.015), d_model, d_ff, seed=8, device="cuda")
    f = ffn.calibrate_ffn(X, W_up, W_down, 0.6, 8, 0.7, 19, 0)
    torch.cuda.synchronize()
    Xd = X.clone()
    Xd[5, 11] = float("nan")                                  # a whole NaN row of Y_up
    Xd[9, :] = 0
    Xd[9, 20] = float("inf")                                   # +-inf / NaN mixtures
    Xd[12, 30] = -3.0e38
    Y_f = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    act_down = ffn.forward(Xd, f, Y_f)
    assert w4.last_error()[0] == w4.OK
    ws = torch.empty(w4.workspace_size(T, d_model, d_ff, 8), dtype=torch.uint8, device="cuda")
    Yu = torch.empty((T, d_ff), dtype=torch.bfloat16, device="cuda")
    w4.linear(Xd, f.up_plain, ws, Yu)
    torch.cuda.synchronize()
    Yu_n = gu.to_np_f32(Yu)
    assert np.isnan(Yu_n[5]).all()                            # the NaN row reaches every column
    Hn = orc.ffn_hidden(Yu_n)
    c = gu.oracle_calib_from_gpu(f.down)
    ref = orc.prep_activation(Hn, c["inv_s"], c["O"], c["J"])
    _compare_prep(ref, act_down, f.down, T)
