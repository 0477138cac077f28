"""Parity at the full 720x1280x61 token count (T = 57600), in the launch
configuration bench.py times (calib_observe, calib_finalize, pack_weight,
prep_act, gemm_dual on the whole tensors), checked on what the oracle can
afford: the calibration scales over all of X (in row chunks), the packed
weight in full, and the activation codes and Y on 1024 seeded sampled rows."""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L", [synth.FULL_UP, synth.FULL_DOWN], ids=lambda L: L.name)
def test_full_size_sampled(L):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    act = w4.alloc_act(L.T, pw)
    Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.prep_act(X, pw, act)
    w4.gemm_dual(act, L.T, pw, Y)
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"

    # calibration over every token, chunked on the host
    run = None
    for r0 in range(0, L.T, 4096):
        run = orc.col_absmax(gu.to_np_f32(X[r0:r0 + 4096]), run)
    np.testing.assert_array_equal(pw.act_scale.cpu().numpy(), run)
    Wn = gu.to_np_f32(W)
    np.testing.assert_array_equal(pw.w_scale.cpu().numpy(), orc.col_absmax(Wn))
    c = gu.oracle_calib_from_gpu(pw)
    np.testing.assert_array_equal(pw.O.cpu().numpy(), c["O"])

    ref_w = orc.pack_weight(Wn, c["s"], c["O"], c["J"], L.layout)
    d = pw.dims
    nb = ref_w["sfb"].shape[1]
    np.testing.assert_array_equal(pw.wq.view(L.d_out, -1).cpu().numpy()[:, :nb * 16], ref_w["wq"])

    rows = synth.sample_rows(L.T, 1024).numpy()
    ridx = torch.from_numpy(rows).cuda()
    ref_a = orc.prep_activation(gu.to_np_f32(X[ridx]), c["inv_s"], c["O"], c["J"])
    np.testing.assert_array_equal(act.aq[ridx].cpu().numpy()[:, :nb * 16], ref_a["aq"])
    sfa = gu.sf_canonical(act.sfa, rows, d.nblk, nb)
    np.testing.assert_array_equal(sfa[:, :nb], ref_a["sfa"])
    np.testing.assert_array_equal(gu.bf16_bits(act.xo[ridx])[:, :L.k], ref_a["xo"])

    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y[ridx]).astype(np.float64), Y_ref, L.name)


def test_full_size_ffn_sampled():
    """The fused FFN at T = 57600 as bench.py --workload ffn runs it (prep, up
    GEMM with the GELU/prep epilogue, down GEMM): the down layer's codes,
    scales and outlier columns on 1024 sampled rows against the oracle's prep
    of bf16(gelu(Y_up)), Y_up from the library's plain up GEMM on those rows
    (rows are independent and each output column accumulates in one fixed K
    order, so it is the value the fused kernel rounded), and Y on those rows
    within the product tolerance."""
    from w4a4_mxfp4_outlier_b200 import ffn
    Lu, Ld = synth.FULL_UP, synth.FULL_DOWN
    X, W_up = gu.gen(Lu)
    W_down = synth.gen_w(Ld.w, Ld.d_out, Ld.d_in, seed=Ld.seed + 1, device="cuda")
    f = ffn.calibrate_ffn(X, W_up, W_down, Lu.alpha, Lu.k, Ld.alpha, Ld.k, Lu.layout)
    Y = torch.empty((Lu.T, Lu.d_in), dtype=torch.bfloat16, device="cuda")
    act_down = ffn.forward(X, f, Y)
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"

    rows = synth.sample_rows(Lu.T, 1024).numpy()
    ridx = torch.from_numpy(rows).cuda()
    Xs = X[ridx].contiguous()
    ws = torch.empty(w4.workspace_size(Xs.shape[0], Lu.d_in, Lu.d_out, Lu.k), dtype=torch.uint8,
                     device="cuda")
    Yu = torch.empty((Xs.shape[0], Lu.d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(Xs, f.up_plain, ws, Yu)
    Hn = orc.ffn_hidden(gu.to_np_f32(Yu))
    c = gu.oracle_calib_from_gpu(f.down)
    ref_a = orc.prep_activation(Hn, c["inv_s"], c["O"], c["J"])
    d = f.down.dims
    nb = ref_a["sfa"].shape[1]
    np.testing.assert_array_equal(act_down.aq[ridx].cpu().numpy()[:, :nb * 16], ref_a["aq"])
    sfa = gu.sf_canonical(act_down.sfa, rows, d.nblk, nb)
    np.testing.assert_array_equal(sfa[:, :nb], ref_a["sfa"])
    np.testing.assert_array_equal(gu.bf16_bits(act_down.xo[ridx])[:, :Ld.k], ref_a["xo"])

    ref_w = orc.pack_weight(gu.to_np_f32(W_down), c["s"], c["O"], c["J"], Lu.layout)
    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y[ridx]).astype(np.float64), Y_ref, "ffn_full_down")


def _channel_groups(d_out: int, n_groups: int, seed: int = 9) -> np.ndarray:
    """Whole 32-row groups of output channels (so 32x32 weight tiles sampled
    this way are the tiles of the full pack), seeded."""
    g = np.sort(np.random.default_rng(seed).choice(d_out // 32, n_groups, replace=False))
    return (g[:, None] * 32 + np.arange(32)[None, :]).reshape(-1)


@pytest.mark.parametrize("L", synth.sweep_layers(), ids=lambda L: L.name)
def test_sweep_sampled(L):
    """Every sweep point at its own size (T = 16384, 5120 -> 13824): k in
    {0, 16, 64, 256} x weight scales {32x1, 32x32, 128x1} x alpha in {0.5, 0.7}
    in bench.py's launch configuration (calibration, pack, prep and GEMM on the
    whole tensors).  Checked on what the oracle affords: the outlier set, the
    packed weight of 16 whole 32-channel groups (512 output channels), the
    activation codes of 512 sampled token rows, and Y on those rows and
    channels."""
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    act = w4.alloc_act(L.T, pw)
    Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.prep_act(X, pw, act)
    w4.gemm_dual(act, L.T, pw, Y)
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"
    c = gu.oracle_calib_from_gpu(pw)
    np.testing.assert_array_equal(pw.O.cpu().numpy(), c["O"])

    chans = _channel_groups(L.d_out, 16)
    cidx = torch.from_numpy(chans).cuda()
    ref_w = orc.pack_weight(gu.to_np_f32(W[cidx]), c["s"], c["O"], c["J"], L.layout)
    d = pw.dims
    nb = ref_w["sfb"].shape[1]
    np.testing.assert_array_equal(pw.wq.view(L.d_out, -1)[cidx].cpu().numpy()[:, :nb * 16],
                                  ref_w["wq"])
    if d.nblk:
        sfb = gu.sf_canonical(pw.sfb, chans, d.nblk, nb)
        np.testing.assert_array_equal(sfb[:, :nb], ref_w["sfb"])
    if L.k:
        np.testing.assert_array_equal(
            gu.bf16_bits(pw.w_hp).reshape(L.d_out, d.k_pad)[chans, :L.k], ref_w["w_hp"])

    rows = synth.sample_rows(L.T, 512).numpy()
    ridx = torch.from_numpy(rows).cuda()
    ref_a = orc.prep_activation(gu.to_np_f32(X[ridx]), c["inv_s"], c["O"], c["J"])
    np.testing.assert_array_equal(act.aq[ridx].cpu().numpy()[:, :nb * 16], ref_a["aq"])
    if d.nblk:
        sfa = gu.sf_canonical(act.sfa, rows, d.nblk, nb)
        np.testing.assert_array_equal(sfa[:, :nb], ref_a["sfa"])
    if L.k:
        np.testing.assert_array_equal(gu.bf16_bits(act.xo[ridx])[:, :L.k], ref_a["xo"])
    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    Ys = gu.to_np_f32(Y[ridx][:, cidx]).astype(np.float64)
    gu.check_tolerance(Ys, Y_ref, L.name)
