"""The FFN pair on the GPU: GELU, packing with permuted rows, and the fused
up-projection epilogue against the oracle; fused and unfused FFN outputs.

The fused epilogue is checked bit for bit against the oracle applied to the
GPU's own (unfused) up-layer output: bf16(acc) is the same value in both
GPU paths (one kernel main loop, the epilogue differs), so from there every
step -- the correctly rounded bf16 GELU, the multiply by inv_s, the MXFP4
encoding -- is a function of that value (a rounding, a float32 product, an
integer decision) that both sides compute alike."""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from w4a4_mxfp4_outlier_b200 import ffn
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

XS = synth.XSpec("student3", 0.3, 6, 8.0, 30.0)


@pytest.mark.parametrize("shift", [0, 1])
def test_gelu_every_bf16(shift):
    # all 65536 inputs, infinities and NaNs included (+inf -> +inf, -inf and NaN -> NaN);
    # the kernel works on bf16 pairs, so each input is checked in the low half
    # (shift 0) and in the high half (shift 1) of its pair -- the same function
    # the fused GEMM epilogue evaluates
    bits = np.roll(np.arange(65536, dtype=np.uint32).astype(np.uint16), shift)
    Y = torch.from_numpy(bits.view(np.int16).reshape(-1, 64)).cuda().view(torch.bfloat16)
    H = ffn.gelu_bf16(Y)
    torch.cuda.synchronize()
    ref = orc.f32_to_bf16_bits(orc.gelu_bf16(orc.bf16_bits_to_f32(bits))).reshape(-1, 64)
    np.testing.assert_array_equal(gu.bf16_bits(H), ref)


@pytest.mark.parametrize("layout", [0, 1, 2])
def test_pack_rows_matches_permuted_pack(layout):
    L = synth.Layer("rows", 64, 512, 368, 0.6, 9, layout, XS, synth.WSpec(0.02), seed=4)
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, layout)
    perm = torch.from_numpy(np.random.default_rng(1).permutation(L.d_out).astype(np.int32)).cuda()
    pr = w4.alloc_packed(L.d_in, L.d_out, L.k, layout)
    pr.s, pr.inv_s, pr.O, pr.jmap = pw.s, pw.inv_s, pw.O, pw.jmap
    import ctypes
    st = w4._pack_weight_rows(W.data_ptr(), W.stride(0), pr.s.data_ptr(), perm.data_ptr(),
                              ctypes.byref(pr.c), None)
    assert st == w4.OK
    torch.cuda.synchronize()
    c = gu.oracle_calib_from_gpu(pw)
    Wp = gu.to_np_f32(W)[perm.cpu().numpy()]
    ref = orc.pack_weight(Wp, c["s"], c["O"], c["J"], layout)
    nb = ref["sfb"].shape[1]
    np.testing.assert_array_equal(pr.wq.view(L.d_out, -1).cpu().numpy()[:, :nb * 16], ref["wq"])
    d = pr.dims
    sfb = gu.sf_canonical(pr.sfb, d.sfb_rows, d.nblk, nb)
    np.testing.assert_array_equal(sfb[:L.d_out, :nb], ref["sfb"])
    np.testing.assert_array_equal(gu.bf16_bits(pr.w_hp).reshape(L.d_out, -1)[:, :L.k], ref["w_hp"])


@pytest.mark.parametrize("layout", [0, 1, 2])
def test_permute_packed_rows_matches_reordered_natural_pack(layout):
    L = synth.Layer("perm", 64, 512, 368, 0.6, 9, layout, XS, synth.WSpec(0.02), seed=4)
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, layout)
    perm = torch.from_numpy(np.random.default_rng(1).permutation(L.d_out).astype(np.int32)).cuda()
    pr = w4.alloc_packed(L.d_in, L.d_out, L.k, layout)
    pr.s, pr.inv_s, pr.O, pr.jmap = pw.s, pw.inv_s, pw.O, pw.jmap
    import ctypes
    st = w4._permute_packed_rows(ctypes.byref(pw.c), perm.data_ptr(), ctypes.byref(pr.c), None)
    assert st == w4.OK
    torch.cuda.synchronize()
    c = gu.oracle_calib_from_gpu(pw)
    ref = orc.pack_weight(gu.to_np_f32(W), c["s"], c["O"], c["J"], layout)
    p = perm.cpu().numpy()
    nb = ref["sfb"].shape[1]
    np.testing.assert_array_equal(pr.wq.view(L.d_out, -1).cpu().numpy()[:, :nb * 16], ref["wq"][p])
    d = pr.dims
    sfb = gu.sf_canonical(pr.sfb, d.sfb_rows, d.nblk, nb)
    np.testing.assert_array_equal(sfb[:L.d_out, :nb], ref["sfb"][p])
    np.testing.assert_array_equal(gu.bf16_bits(pr.w_hp).reshape(L.d_out, -1)[:, :L.k], ref["w_hp"][p])
    # in place is refused
    assert w4._permute_packed_rows(ctypes.byref(pw.c), perm.data_ptr(), ctypes.byref(pw.c),
                                   None) == w4.ERR_INVALID_ARG


FFN_CASES = [
    # T, d_model, d_ff, k_up, k_down, layout
    (300, 512, 1376, 8, 19, 0),      # pair GEMM; ragged d_ff; kj_pad of the down layer > d_ff
    (100, 256, 640, 4, 32, 2),       # single-CTA GEMM (T <= 128), 128x1 stripes
    (520, 1024, 2048, 16, 0, 1),     # no outliers in the down layer, 32x32 tiles
    (300, 512, 1376, 8, 19, 1),      # 32x32 tiles with a non-trivial channel order
    # d_ff a multiple of 384: the unfused path's up GEMM runs on 256 x 384
    # pair tiles, the fused one on 256 x 256 (the two must agree bit for bit)
    (300, 512, 1536, 8, 19, 0),      # outliers of the down layer in the last tile's half 1
    (520, 1024, 768, 16, 0, 1),      # no outliers in the down layer, 32x32 tiles
    (257, 256, 1152, 4, 64, 2),      # ragged M tile, 128x1 stripes
    (300, 512, 768, 8, 300, 0),      # down layer with 16 MX blocks: whole code groups past it
]


def _make_ffn(T, d_model, d_ff, k_up, k_down, layout):
    Lx = synth.Layer("ffn_up", T, d_model, d_ff, 0.6, k_up, layout, XS, synth.WSpec(0.02), seed=7)
    X, W_up = gu.gen(Lx)
    W_down = synth.gen_w(synth.WSpec(0.015), d_model, d_ff, seed=8, device="cuda")
    f = ffn.calibrate_ffn(X, W_up, W_down, 0.6, k_up, 0.7, k_down, layout)
    torch.cuda.synchronize()
    return X, W_up, W_down, f


@pytest.mark.parametrize("case", FFN_CASES, ids=lambda c: "T%d_%dx%d_k%d_%d_l%d" % c)
def test_fused_epilogue_matches_oracle_and_unfused(case):
    T, d_model, d_ff, k_up, k_down, layout = case
    X, W_up, W_down, f = _make_ffn(*case)
    Y_f = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    act_down = ffn.forward(X, f, Y_f)
    Y_u = torch.empty_like(Y_f)
    H = ffn.forward_unfused(X, f, Y_u)
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)
    # the oracle's down-layer prep of bf16(gelu(Y_up)), Y_up from the GPU's up GEMM
    ws = torch.empty(w4.workspace_size(T, d_model, d_ff, k_up), dtype=torch.uint8, device="cuda")
    Yu = torch.empty((T, d_ff), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, f.up_plain, ws, Yu)
    Hn = orc.ffn_hidden(gu.to_np_f32(Yu))
    np.testing.assert_array_equal(orc.f32_to_bf16_bits(Hn), gu.bf16_bits(H))
    c = gu.oracle_calib_from_gpu(f.down)
    ref = orc.prep_activation(Hn, c["inv_s"], c["O"], c["J"])
    d = f.down.dims
    nb = ref["sfa"].shape[1]
    aq = act_down.aq.cpu().numpy()
    np.testing.assert_array_equal(aq[:, :nb * 16], ref["aq"], err_msg="codes")
    assert not aq[:, nb * 16:].any()
    if d.nblk:
        sfa = gu.sf_canonical(act_down.sfa, T, d.nblk, nb)
        np.testing.assert_array_equal(sfa[:, :nb], ref["sfa"], err_msg="scales")
        assert not sfa[:, nb:].any()
    xo = gu.bf16_bits(act_down.xo)
    np.testing.assert_array_equal(xo[:, :k_down], ref["xo"], err_msg="outlier columns")
    assert not xo[:, k_down:].any()
    # and the whole FFN: fused == unfused, bit for bit
    assert torch.equal(Y_f.view(torch.int16), Y_u.view(torch.int16))


# ---------------------------------------------------------------------------
# The down layer's Y against an oracle chain that starts from X
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", [(300, 512, 1376, 8, 19, 0), (300, 512, 1376, 8, 19, 1)],
                         ids=lambda c: "T%d_%dx%d_k%d_%d_l%d" % c)
def test_ffn_down_output_against_oracle_chain_from_x(case):
    """Y of the whole fused FFN against the oracle run from X alone (its own
    up product in float64, GELU, down prep, down product), with the
    library's calibration (s, O, J) on both layers.  The GPU's bf16 Y_up may
    lie anywhere within the up layer's tolerance of the oracle's; that band,
    rounded outward to bf16, is carried through GELU, the smoothing multiply,
    the MXFP4 quantiser and the down product (tests/ffn_bounds.py), giving for
    each output an interval that contains every down product such a Y_up can
    produce.  The GPU's Y must lie within the down layer's tolerance of that
    interval."""
    from tests import ffn_bounds as fb
    T, d_model, d_ff, k_up, k_down, layout = case
    X, W_up, W_down, f = _make_ffn(*case)
    Y = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    ffn.forward(X, f, Y)
    assert w4.last_error()[0] == w4.OK
    cu, cd = gu.oracle_calib_from_gpu(f.up_plain), gu.oracle_calib_from_gpu(f.down)
    wu = orc.pack_weight(gu.to_np_f32(W_up), cu["s"], cu["O"], cu["J"], layout)
    au = orc.prep_activation(gu.to_np_f32(X), cu["inv_s"], cu["O"], cu["J"])
    Yu = orc.dual_branch_product(au["aq"], au["sfa"], au["xo"], wu["wq"], wu["sfb"], wu["w_hp"])
    Ylo, Yhi = fb.down_interval(Yu, fb.up_tolerance(Yu), cd, gu.to_np_f32(W_down), layout)
    Yg = gu.to_np_f32(Y).astype(np.float64)
    rms = float(np.sqrt(np.mean((0.5 * (Ylo + Yhi)) ** 2)))
    outside = np.maximum(np.maximum(Ylo - Yg, Yg - Yhi), 0.0)
    bound = 8e-3 * np.maximum(np.abs(Ylo), np.abs(Yhi)) + 1e-3 * rms
    assert (outside <= bound).all(), f"{int((outside > bound).sum())} outputs outside, worst " \
        f"{float((outside / bound).max()):.2f} of the bound"
    # the interval says something: its typical width is a fraction of the outputs
    assert float(np.median(Yhi - Ylo)) < 0.5 * rms
