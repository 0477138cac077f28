"""Seeded random shapes through the whole path (calibration, packing, prep,
GEMM) against the oracle: T from 1 to 700 (single-CTA and pair GEMM, ragged
tiles), d_in from 8 to 6000 in steps of 8, d_out from 16 to 1200 in steps of
16, k from 0 to d_in, all three weight-scale layouts and a spread of alpha.
The codes, scales, outlier columns and packed weight bit for bit; Y within
the product tolerance.  And random FFN pairs: fused == unfused bit for bit,
the fused epilogue's codes against the oracle."""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from w4a4_mxfp4_outlier_b200 import ffn
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _cases(n=80, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T = int(rng.choice([1, 7, 64, 128, 129, 255, 300, 513, 700]))
        d_in = int(rng.integers(1, 751)) * 8
        d_out = int(rng.integers(1, 76)) * 16
        k = int(rng.choice([0, 1, 3, 16, 33, d_in // 7, d_in]))
        k = min(k, d_in)
        layout = int(rng.integers(0, 3))
        alpha = float(rng.choice([0.3, 0.5, 0.6, 0.8]))
        planted = int(min(d_in, rng.integers(0, 24)))
        xs = synth.XSpec("student3", 0.3, planted, 8.0, 30.0)
        out.append(synth.Layer(f"rand{i}_T{T}_{d_in}x{d_out}_k{k}_l{layout}", T, d_in, d_out, alpha,
                               k, layout, xs, synth.WSpec(0.02), seed=100 + i))
    return out


def _cases384(n=16, seed=2025):
    """Shapes that run on the 384-column pair tile: d_out a multiple of 384, T > 128."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T = int(rng.choice([129, 200, 256, 257, 511, 700]))
        d_in = int(rng.integers(1, 400)) * 8
        d_out = int(rng.integers(1, 5)) * 384
        k = min(int(rng.choice([0, 1, 17, 64, 100, d_in])), d_in)
        layout = int(rng.integers(0, 3))
        alpha = float(rng.choice([0.4, 0.6, 0.7]))
        xs = synth.XSpec("student3", 0.3, int(min(d_in, rng.integers(0, 16))), 8.0, 30.0)
        out.append(synth.Layer(f"rand384_{i}_T{T}_{d_in}x{d_out}_k{k}_l{layout}", T, d_in, d_out,
                               alpha, k, layout, xs, synth.WSpec(0.02), seed=300 + i))
    return out


@pytest.mark.parametrize("L", _cases() + _cases384(), ids=lambda L: L.name)
def test_random_shape_parity(L):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    act = w4.alloc_act(L.T, pw)
    w4.prep_act(X, pw, act)
    Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.gemm_dual(act, L.T, pw, Y)
    torch.cuda.synchronize()
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)

    c = gu.oracle_calib_from_gpu(pw)
    np.testing.assert_array_equal(pw.O.cpu().numpy(), c["O"])
    Xn, Wn = gu.to_np_f32(X), gu.to_np_f32(W)
    ref_w = orc.pack_weight(Wn, c["s"], c["O"], c["J"], L.layout)
    ref_a = orc.prep_activation(Xn, c["inv_s"], c["O"], c["J"])
    d = pw.dims
    nb = ref_a["sfa"].shape[1]
    np.testing.assert_array_equal(pw.wq.view(L.d_out, -1).cpu().numpy()[:, :nb * 16], ref_w["wq"])
    np.testing.assert_array_equal(act.aq.cpu().numpy()[:, :nb * 16], ref_a["aq"])
    if d.nblk:
        np.testing.assert_array_equal(gu.sf_canonical(pw.sfb, d.sfb_rows, d.nblk, nb)[:L.d_out, :nb],
                                      ref_w["sfb"])
        np.testing.assert_array_equal(gu.sf_canonical(act.sfa, L.T, d.nblk, nb)[:, :nb], ref_a["sfa"])
    if L.k:
        np.testing.assert_array_equal(gu.bf16_bits(act.xo)[:, :L.k], ref_a["xo"])
        np.testing.assert_array_equal(gu.bf16_bits(pw.w_hp).reshape(L.d_out, d.k_pad)[:, :L.k],
                                      ref_w["w_hp"])
    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y).astype(np.float64), Y_ref, L.name)


def _ffn_cases(n=24, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T = int(rng.choice([5, 128, 200, 333, 600]))
        d_model = int(rng.integers(2, 97)) * 16
        d_ff = int(rng.integers(2, 161)) * 16
        k_up = int(min(d_model, rng.choice([0, 4, 16, 40])))
        k_down = int(min(d_ff, rng.choice([0, 7, 19, 64, d_ff])))
        layout = int(rng.integers(0, 3))
        out.append((f"ffn{i}_T{T}_{d_model}x{d_ff}_k{k_up}_{k_down}_l{layout}", T, d_model, d_ff,
                    k_up, k_down, layout, 100 + i))
    # d_ff a multiple of 384 with T > 128: the unfused up GEMM on 384-wide
    # tiles against the fused one on 256-wide tiles
    for i in range(8):
        T = int(rng.choice([129, 200, 333, 600]))
        d_model = int(rng.integers(2, 65)) * 16
        d_ff = int(rng.integers(1, 5)) * 384
        k_up = int(min(d_model, rng.choice([0, 4, 16, 40])))
        k_down = int(min(d_ff, rng.choice([0, 7, 19, 64, 300, d_ff])))
        layout = int(rng.integers(0, 3))
        out.append((f"ffn384_{i}_T{T}_{d_model}x{d_ff}_k{k_up}_{k_down}_l{layout}", T, d_model,
                    d_ff, k_up, k_down, layout, 200 + i))
    return out


@pytest.mark.parametrize("case", _ffn_cases(), ids=lambda c: c[0])
def test_random_ffn_parity(case):
    _, T, d_model, d_ff, k_up, k_down, layout, seed = case
    xs = synth.XSpec("student3", 0.3, min(d_model, 6), 8.0, 30.0)
    Lx = synth.Layer("rffn", T, d_model, d_ff, 0.6, k_up, layout, xs, synth.WSpec(0.02), seed=seed)
    X, W_up = gu.gen(Lx)
    W_down = synth.gen_w(synth.WSpec(0.015), d_model, d_ff, seed=seed + 50, device="cuda")
    f = ffn.calibrate_ffn(X, W_up, W_down, 0.6, k_up, 0.7, k_down, layout)
    Y_f = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    act_down = ffn.forward(X, f, Y_f)
    Y_u = torch.empty_like(Y_f)
    ffn.forward_unfused(X, f, Y_u)
    torch.cuda.synchronize()
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)
    assert torch.equal(Y_f.view(torch.int16), Y_u.view(torch.int16))
    # the fused epilogue's codes against the oracle's prep of bf16(gelu(Y_up))
    ws = torch.empty(w4.workspace_size(T, d_model, d_ff, k_up), dtype=torch.uint8, device="cuda")
    Yu = torch.empty((T, d_ff), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, f.up_plain, ws, Yu)
    c = gu.oracle_calib_from_gpu(f.down)
    ref = orc.prep_activation(orc.ffn_hidden(gu.to_np_f32(Yu)), c["inv_s"], c["O"], c["J"])
    d = f.down.dims
    nb = ref["sfa"].shape[1]
    np.testing.assert_array_equal(act_down.aq.cpu().numpy()[:, :nb * 16], ref["aq"])
    if d.nblk:
        np.testing.assert_array_equal(gu.sf_canonical(act_down.sfa, T, d.nblk, nb)[:, :nb], ref["sfa"])
    if k_down:
        np.testing.assert_array_equal(gu.bf16_bits(act_down.xo)[:, :k_down], ref["xo"])


@pytest.mark.parametrize("L", _cases()[::4], ids=lambda L: L.name)
def test_random_shape_variants(L):
    """The same layer through the other entry points gives the same bits as
    linear: a checkpoint round trip, the no-allocation entry point (where the
    problem fits its scratch array) and strided X and Y rows."""
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, pw, ws, Y)
    # checkpoint round trip
    pl = w4.packed_from_bytes(w4.packed_to_bytes(pw))
    Y2 = torch.empty_like(Y)
    w4.linear(X, pl, ws, Y2)
    # strided rows
    Xs = torch.zeros((L.T, L.d_in + 24), dtype=torch.bfloat16, device="cuda")
    Xs[:, :L.d_in] = X
    Ys = torch.zeros((L.T, L.d_out + 48), dtype=torch.bfloat16, device="cuda")
    w4.linear(Xs[:, :L.d_in], pw, ws, Ys[:, :L.d_out])
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(Y.view(torch.int16), Ys[:, :L.d_out].contiguous().view(torch.int16))
    assert not Ys[:, L.d_out:].any()
    if ws.numel() <= w4.NOALLOC_SCRATCH_BYTES:
        Y3 = torch.empty_like(Y)
        w4.linear_noalloc(X, pw, Y3)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y3.view(torch.int16))
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)


def _topk_cases(n=30, seed=5):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d_in = int(rng.integers(1, 2049)) * 8
        k = int(rng.choice([0, 1, 2, 31, 64, 257, d_in // 2, d_in - 1, d_in]))
        k = max(0, min(k, d_in))
        nvals = int(rng.choice([1, 2, 3, 17, 1000]))
        out.append((f"topk{i}_d{d_in}_k{k}_v{nvals}", d_in, k, nvals, 300 + i))
    return out


@pytest.mark.parametrize("case", _topk_cases(), ids=lambda c: c[0])
def test_random_topk_with_ties(case):
    """The device top-k (radix select, ties to the lower column) against the
    oracle's stable sort, on scores with many exact ties: with alpha = 0.5 and
    weight magnitudes equal to the activation magnitudes, s = 1 and the score
    is the activation magnitude itself."""
    _, d_in, k, nvals, seed = case
    rng = np.random.default_rng(seed)
    vals = np.concatenate([[0.0], rng.uniform(1e-3, 50.0, nvals - 1)]).astype(np.float32)
    act = torch.from_numpy(vals[rng.integers(0, nvals, d_in)]).cuda()
    wsc = act.clone()
    f = lambda: torch.empty(d_in, device="cuda")
    s, inv_s, score = f(), f(), f()
    O = torch.empty(max(k, 1), dtype=torch.int32, device="cuda")
    J = torch.empty(max(d_in - k, 1), dtype=torch.int32, device="cuda")
    w4.calib_finalize(act, wsc, 0.5, k, s, inv_s, score, O if k else None, J if k < d_in else None)
    torch.cuda.synchronize()
    sc = score.cpu().numpy()
    assert np.array_equal(sc, act.cpu().numpy())
    Oref, Jref = orc.select_outliers(sc, k)
    if k:
        np.testing.assert_array_equal(O.cpu().numpy()[:k], Oref)
    if k < d_in:
        np.testing.assert_array_equal(J.cpu().numpy()[:d_in - k], Jref)


def test_prep_special_values():
    """Prep of rows that are all zero, subnormal, huge (near the bf16 maximum
    after smoothing) or mixed in sign and magnitude, with a layer calibrated
    on ordinary data: codes, scales and outliers bit for bit."""
    L = synth.Layer("special", 64, 512, 256, 0.5, 12, 0, synth.XSpec("student3", 0.3, 6, 8.0, 30.0),
                    synth.WSpec(0.02), seed=21)
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    rng = np.random.default_rng(9)
    rows = []
    rows.append(np.zeros(512))                                         # all zero
    rows.append(np.full(512, -0.0))                                    # negative zeros
    rows.append(rng.choice([-1, 1], 512) * 2.0 ** rng.integers(-133, -126, 512))   # bf16 subnormals
    rows.append(rng.choice([-1, 1], 512) * rng.uniform(1e30, 3e33, 512))           # huge
    rows.append(np.where(rng.random(512) < 0.5, 0.0, rng.normal(0, 1e-20, 512)))   # tiny, sparse
    rows.append(rng.normal(0, 1, 512) * 10.0 ** rng.integers(-30, 30, 512))        # wild magnitudes
    while len(rows) < 64:
        rows.append(rng.normal(0, 0.3, 512))
    Xs = torch.from_numpy(np.stack(rows).astype(np.float32)).to(torch.bfloat16).cuda()
    act = w4.alloc_act(64, pw)
    w4.prep_act(Xs, pw, act)
    torch.cuda.synchronize()
    c = gu.oracle_calib_from_gpu(pw)
    ref = orc.prep_activation(gu.to_np_f32(Xs), c["inv_s"], c["O"], c["J"])
    d = pw.dims
    nb = ref["sfa"].shape[1]
    np.testing.assert_array_equal(act.aq.cpu().numpy()[:, :nb * 16], ref["aq"])
    np.testing.assert_array_equal(gu.sf_canonical(act.sfa, 64, d.nblk, nb)[:, :nb], ref["sfa"])
    np.testing.assert_array_equal(gu.bf16_bits(act.xo)[:, :L.k], ref["xo"])
