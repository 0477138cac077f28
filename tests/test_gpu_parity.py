"""GPU parity: every stage of the library against the CPU oracle.

Integer and byte outputs (scales, codes, gathered outlier columns, index
lists) must match bit for bit; Y must satisfy
|Y_gpu - Y_ref| <= 8e-3 |Y_ref| + 1e-3 rms(Y_ref) element by element, Y_ref
being the oracle's float64 product of its own dequantised operands.

The smoothing factor is a float64 pow on both sides; the two libms may
differ in the last bit of the float64 result, so s is compared within one
float32 ulp and the downstream stages (score, O, packing, prep) are fed the
library's s / inv_s so they can be compared bit for bit.
"""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

TINY = synth.TINY
RAGGED = synth.Layer("ragged", 200, 136, 368, 0.6, 3, 0, synth.XSpec("student3", 0.3, 4, 8.0, 30.0),
                     synth.WSpec(0.02))
RAGGED32 = RAGGED.with_(name="ragged_32x32", layout=1, k=11)
RAGGED128 = RAGGED.with_(name="ragged_128x1", layout=2, k=7, d_in=904)   # partial last stripe
K0 = TINY.with_(name="k0", k=0)
KFULL = synth.Layer("kfull", 300, 64, 272, 0.5, 64, 0, synth.X_TINY, synth.WSpec(0.02))
T1 = TINY.with_(name="T1", T=1)
MID = synth.Layer("mid_k256_32x32", 640, 5120, 1024, 0.7, 256, 1, synth.X_UP, synth.W_UP)
FFN0 = synth.FFN0
FFN2 = synth.FFN2

SINGLE = RAGGED.with_(name="ragged_T100_single_cta", T=100, k=5)   # T <= 128: single-CTA GEMM

MID128 = MID.with_(name="mid_k64_128x1", layout=2, k=64)

SMALL = [TINY, RAGGED, RAGGED32, RAGGED128, K0, KFULL, T1, SINGLE]

# the 384-column pair tile (d_out a multiple of 384, T > 128): ragged M tile,
# ragged last bf16 K tile (k = 37), one to three N tiles, all three weight
# scale layouts, no MXFP4 columns at all (k = d_in) and no outliers (k = 0)
TILE384 = [
    synth.Layer("tile384_T300_k37", 300, 1024, 768, 0.6, 37, 0, synth.X_UP, synth.W_UP),
    synth.Layer("tile384_T129_32x32_k0", 129, 512, 1152, 0.5, 0, 1, synth.X_UP, synth.W_UP),
    synth.Layer("tile384_T520_128x1_k64", 520, 2048, 384, 0.7, 64, 2, synth.X_UP, synth.W_UP),
    synth.Layer("tile384_kfull", 300, 64, 384, 0.5, 64, 0, synth.X_TINY, synth.WSpec(0.02)),
]

# the prep kernel's launch shapes: block-per-lane form with 2 thread groups
# (192 blocks; with the 6-slot ring at d_in 6144 and the 18-slot ring for
# short rows at 5440; 6 and 3 groups on short rows are the small shapes and
# FFN0), with 1 group at its 480-block limit, with more outlier pairs
# than blocks (k = 900) and more than its 480 lanes (k = 1500: the extra pairs
# loop); the 8-columns-per-lane form past 480 blocks (d_in = 16384, also with
# 128x1 stripes)
G2 = synth.Layer("prep_g2_d6144", 200, 6144, 272, 0.6, 20, 0, synth.X_UP, synth.W_UP)
G2N = synth.Layer("prep_g2_d5440", 230, 5440, 256, 0.6, 20, 0, synth.X_UP, synth.W_UP)
B480 = synth.Layer("prep_b480_d15360", 150, 15360, 256, 0.6, 16, 0, synth.X_UP, synth.W_UP)
XOWIDE = synth.Layer("prep_xo_k900", 160, 1024, 256, 0.5, 900, 0, synth.X_UP, synth.W_UP)
XOLOOP = synth.Layer("prep_xo_k1500", 100, 2048, 256, 0.5, 1500, 0, synth.X_UP, synth.W_UP)
WIDE = synth.Layer("prep_wide_d16384", 300, 16384, 256, 0.6, 40, 0, synth.X_UP, synth.W_UP)
WIDE128 = WIDE.with_(name="prep_wide_d16384_128x1", layout=2, k=24)
PREP_SHAPES = [G2, G2N, B480, XOWIDE, XOLOOP, WIDE, WIDE128]


def _calibrate(L):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    torch.cuda.synchronize()
    return X, W, pw


# ---------------------------------------------------------------------------
# Encoder: every finite bfloat16 value through the prep kernel
# ---------------------------------------------------------------------------
def _manual_pw(d_in, k, inv_s, O, J):
    pw = w4.alloc_packed(d_in, 16, k)
    pw.inv_s.copy_(torch.from_numpy(inv_s))
    if k:
        pw.O.copy_(torch.from_numpy(O.astype(np.int32)))
    if d_in - k:
        pw.jmap.copy_(torch.from_numpy(J.astype(np.int32)))
    return pw


@pytest.mark.parametrize("variant", ["identity", "random_inv_s", "shuffled"])
def test_prep_encodes_every_bf16_value(variant):
    bits = np.arange(65536, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    vals = bits[finite].astype(np.uint16)
    rng = np.random.default_rng(0)
    if variant == "shuffled":
        vals = rng.permutation(vals)
    d_in = 512
    T = -(-vals.size // d_in)
    Xb = np.zeros(T * d_in, np.uint16)
    Xb[:vals.size] = vals
    Xb = Xb.reshape(T, d_in)
    X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
    inv_s = np.ones(d_in, np.float32)
    if variant == "random_inv_s":
        inv_s = rng.uniform(0.01, 1.0, d_in).astype(np.float32)   # no overflow to inf
    O = np.array([5, 100, 511], np.int32) if variant != "identity" else np.zeros(0, np.int32)
    J = np.setdiff1d(np.arange(d_in), O).astype(np.int32)
    pw = _manual_pw(d_in, len(O), inv_s, O, J)
    act = w4.alloc_act(T, pw)
    w4.prep_act(X, pw, act)
    torch.cuda.synchronize()
    Xf = orc.bf16_bits_to_f32(Xb)
    ref = orc.prep_activation(Xf, inv_s, O, J)
    _compare_prep(ref, act, pw, T)


def _compare_prep(ref, act, pw, T):
    d = pw.dims
    nb_ref = ref["sfa"].shape[1]
    aq = act.aq.cpu().numpy()
    np.testing.assert_array_equal(aq[:, :nb_ref * 16], ref["aq"], err_msg="E2M1 codes")
    assert not aq[:, nb_ref * 16:].any(), "code padding must be zero"
    if d.nblk:
        sfa = gu.sf_canonical(act.sfa, T, d.nblk, nb_ref)
        np.testing.assert_array_equal(sfa[:, :nb_ref], ref["sfa"], err_msg="E8M0 scales")
        assert not sfa[:, nb_ref:].any(), "padding blocks must have scale code 0"
    xo = gu.bf16_bits(act.xo)
    np.testing.assert_array_equal(xo[:, :pw.k], ref["xo"], err_msg="gathered outlier columns")
    assert not xo[:, pw.k:].any(), "outlier padding must be zero"


# ---------------------------------------------------------------------------
# Calibration
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L", SMALL + [FFN0, FFN2], ids=lambda L: L.name)
def test_calibration_parity(L):
    X, W, pw = _calibrate(L)
    Xn, Wn = gu.to_np_f32(X), gu.to_np_f32(W)
    act = orc.col_absmax(Xn)
    wsc = orc.col_absmax(Wn)
    np.testing.assert_array_equal(pw.act_scale.cpu().numpy(), act)
    np.testing.assert_array_equal(pw.w_scale.cpu().numpy(), wsc)
    s_ref, inv_ref = orc.smoothing_factors(act, wsc, L.alpha)
    s_gpu = pw.s.cpu().numpy()
    ulp = np.abs(s_gpu.view(np.int32).astype(np.int64) - s_ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1, f"s differs by {ulp.max()} ulp"
    inv_gpu = pw.inv_s.cpu().numpy()
    np.testing.assert_array_equal(inv_gpu, (1.0 / s_gpu.astype(np.float64)).astype(np.float32))
    # the score by its definition, on the smoothed activations, with the library's inv_s
    np.testing.assert_array_equal(pw.score.cpu().numpy(), orc.outlier_scores(Xn, inv_gpu))
    c = gu.oracle_calib_from_gpu(pw)
    np.testing.assert_array_equal(pw.O.cpu().numpy(), c["O"])
    np.testing.assert_array_equal(pw.jmap.cpu().numpy(), c["J"])


def test_calibration_multi_batch_running_max():
    L = RAGGED
    X, W = gu.gen(L)
    X2 = (X.float() * 1.5).to(torch.bfloat16)
    pw = w4.calibrate([X, X2[:77]], W, L.alpha, L.k)
    torch.cuda.synchronize()
    ref = orc.col_absmax(gu.to_np_f32(X2[:77]), orc.col_absmax(gu.to_np_f32(X)))
    np.testing.assert_array_equal(pw.act_scale.cpu().numpy(), ref)


@pytest.mark.parametrize("T,d_out,d_in", [(200, 368, 136), (0, 96, 64), (300, 0, 64),
                                           (57, 1000 - 8, 5120), (4096, 32, 8)])
def test_calibration_layer_call(T, d_out, d_in):
    """X and W in one launch: the values of two single-matrix calls, and of the
    column absmax by its definition; reset = 0 keeps the running maximum."""
    g = torch.Generator().manual_seed(T * 7 + d_out)
    X = (torch.randn(T, d_in, generator=g) * 3).to(torch.bfloat16).cuda()
    W = (torch.randn(d_out, d_in, generator=g) * 0.05).to(torch.bfloat16).cuda()
    f = lambda: torch.full((d_in,), 7.0, device="cuda")
    a1, w1, a2, w2 = f(), f(), f(), f()
    w4.calib_observe_layer(X, W, a1, w1, reset=True)
    w4.calib_observe(X, a2, reset=True)
    w4.calib_observe(W, w2, reset=True)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2) and torch.equal(w1, w2)
    np.testing.assert_array_equal(a1.cpu().numpy(), orc.col_absmax(gu.to_np_f32(X)))
    np.testing.assert_array_equal(w1.cpu().numpy(), orc.col_absmax(gu.to_np_f32(W)))
    # running maximum: a second call without reset on half-size inputs changes nothing
    w4.calib_observe_layer((X.float() * 0.5).to(torch.bfloat16), (W.float() * 0.5).to(torch.bfloat16),
                           a1, w1, reset=False)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2) and torch.equal(w1, w2)


def test_topk_ties_go_to_lower_index():
    d_in, k = 64, 5
    act = torch.ones(d_in, device="cuda")
    act[[3, 9, 20, 40, 41, 50]] = 8.0       # six equal maxima, k = 5: index 50 loses
    wsc = torch.full((d_in,), 0.1, device="cuda")
    f = lambda: torch.empty(d_in, device="cuda")
    s, inv_s, score = f(), f(), f()
    O = torch.empty(k, dtype=torch.int32, device="cuda")
    J = torch.empty(d_in - k, dtype=torch.int32, device="cuda")
    w4.calib_finalize(act, wsc, 0.5, k, s, inv_s, score, O, J)
    torch.cuda.synchronize()
    assert O.cpu().tolist() == [3, 9, 20, 40, 41]
    assert sorted(J.cpu().tolist() + O.cpu().tolist()) == list(range(d_in))


# ---------------------------------------------------------------------------
# Weight packing
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L", SMALL + [MID, MID128, FFN0] + PREP_SHAPES, ids=lambda L: L.name)
def test_pack_parity(L):
    X, W, pw = _calibrate(L)
    c = gu.oracle_calib_from_gpu(pw)
    ref = orc.pack_weight(gu.to_np_f32(W), c["s"], c["O"], c["J"], L.layout)
    d = pw.dims
    nb_ref = ref["sfb"].shape[1]
    wq = pw.wq.view(L.d_out, -1).cpu().numpy()
    np.testing.assert_array_equal(wq[:, :nb_ref * 16], ref["wq"])
    assert not wq[:, nb_ref * 16:].any()
    if d.nblk:
        sfb = gu.sf_canonical(pw.sfb, d.sfb_rows, d.nblk, nb_ref)
        np.testing.assert_array_equal(sfb[:L.d_out, :nb_ref], ref["sfb"])
        assert not sfb[L.d_out:].any()
        tail = nb_ref
        if L.layout == w4.SF_128x1_KMAJOR:
            # padding blocks inside the last, partial stripe carry its code
            tail = -(-nb_ref // 4) * 4
            for b in range(nb_ref, tail):
                np.testing.assert_array_equal(sfb[:L.d_out, b], sfb[:L.d_out, nb_ref - 1])
        assert not sfb[:, tail:].any()
    w_hp = gu.bf16_bits(pw.w_hp).reshape(L.d_out, d.k_pad)
    np.testing.assert_array_equal(w_hp[:, :L.k], ref["w_hp"])
    assert not w_hp[:, L.k:].any()


# ---------------------------------------------------------------------------
# Activation preparation
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L", SMALL + [FFN0, FFN2] + PREP_SHAPES, ids=lambda L: L.name)
def test_prep_parity(L):
    X, W, pw = _calibrate(L)
    c = gu.oracle_calib_from_gpu(pw)
    act = w4.alloc_act(L.T, pw)
    w4.prep_act(X, pw, act)
    torch.cuda.synchronize()
    ref = orc.prep_activation(gu.to_np_f32(X), c["inv_s"], c["O"], c["J"])
    _compare_prep(ref, act, pw, L.T)


def test_prep_row_stride():
    L = RAGGED
    X, W, pw = _calibrate(L)
    big = torch.zeros((L.T, L.d_in + 24), dtype=torch.bfloat16, device="cuda")
    big[:, :L.d_in] = X
    a1, a2 = w4.alloc_act(L.T, pw), w4.alloc_act(L.T, pw)
    w4.prep_act(X, pw, a1)
    w4.prep_act(big[:, :L.d_in], pw, a2)
    torch.cuda.synchronize()
    assert torch.equal(a1.aq, a2.aq) and torch.equal(a1.xo, a2.xo)
    d = pw.dims
    # rows >= T of the scale buffer are padding the kernel does not write
    np.testing.assert_array_equal(gu.sf_canonical(a1.sfa, L.T, d.nblk, d.nblk),
                                  gu.sf_canonical(a2.sfa, L.T, d.nblk, d.nblk))


# ---------------------------------------------------------------------------
# Dual-branch GEMM and the whole online layer
# ---------------------------------------------------------------------------
def _linear(X, pw, T, d_out):
    ws = torch.empty(w4.workspace_size(T, pw.d_in, d_out, pw.k), dtype=torch.uint8, device="cuda")
    Y = torch.empty((T, d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, pw, ws, Y)
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"
    return Y


@pytest.mark.parametrize("L", SMALL + [MID, MID128] + TILE384, ids=lambda L: L.name)
def test_linear_parity_full_output(L):
    X, W, pw = _calibrate(L)
    Y = _linear(X, pw, L.T, L.d_out)
    c = gu.oracle_calib_from_gpu(pw)
    Xn, Wn = gu.to_np_f32(X), gu.to_np_f32(W)
    ref_w = orc.pack_weight(Wn, c["s"], c["O"], c["J"], L.layout)
    ref_a = orc.prep_activation(Xn, c["inv_s"], c["O"], c["J"])
    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y).astype(np.float64), Y_ref, L.name)
    exact = Xn.astype(np.float64) @ Wn.astype(np.float64).T
    assert gu.snr_db(Y_ref, exact) > 10.0


@pytest.mark.parametrize("L", [FFN0, FFN2], ids=lambda L: L.name)
def test_linear_parity_sampled_rows(L):
    X, W, pw = _calibrate(L)
    Y = _linear(X, pw, L.T, L.d_out)
    rows = synth.sample_rows(L.T, 1024).numpy()
    c = gu.oracle_calib_from_gpu(pw)
    Xn = gu.to_np_f32(X[torch.from_numpy(rows).cuda()])
    ref_w = orc.pack_weight(gu.to_np_f32(W), c["s"], c["O"], c["J"], L.layout)
    ref_a = orc.prep_activation(Xn, c["inv_s"], c["O"], c["J"])
    Y_ref = orc.dual_branch_product(ref_a["aq"], ref_a["sfa"], ref_a["xo"], ref_w["wq"],
                                    ref_w["sfb"], ref_w["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y)[rows].astype(np.float64), Y_ref, L.name)


_TILE256_CHILD = """
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
from tests import test_gpu_parity as t
for i, L in enumerate(t.TILE384):
    X, W, pw = t._calibrate(L)
    Y = t._linear(X, pw, L.T, L.d_out)
    np.save(sys.argv[2] + f"/y{i}.npy", Y.view(torch.int16).cpu().numpy())
"""


def test_tile_widths_give_the_same_bits(tmp_path):
    """The 256 x 384 pair tile against the 256 x 256 one on the same inputs:
    W4A4_PAIR_TILE_N=256 is read once per process, so the 256-wide results
    come from a child process."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, W4A4_PAIR_TILE_N="256")
    r = subprocess.run([sys.executable, "-c", _TILE256_CHILD, root, str(tmp_path)], env=env,
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    for i, L in enumerate(TILE384):
        X, W, pw = _calibrate(L)
        Y = _linear(X, pw, L.T, L.d_out)
        y256 = np.load(tmp_path / f"y{i}.npy")
        assert np.array_equal(Y.view(torch.int16).cpu().numpy(), y256), L.name


def test_empty_token_batch_is_a_no_op():
    """T = 0 through every online call and the single-matrix calibration:
    OK, nothing enqueued that touches memory, and the buffers (filled with a
    sentinel) unchanged; the next call on the same buffers is still right."""
    L = RAGGED
    X, W, pw = _calibrate(L)
    X0 = X[:0]
    ws = torch.full((w4.workspace_size(L.T, L.d_in, L.d_out, L.k),), 0x5A, dtype=torch.uint8,
                    device="cuda")
    Y = torch.full((L.T, L.d_out), 3.0, dtype=torch.bfloat16, device="cuda")
    act = w4.alloc_act(L.T, pw)
    for t in (act.aq, act.sfa):
        t.fill_(0x5A)
    act.xo.fill_(3.0)
    snap = [t.clone() for t in (ws, Y, act.aq, act.sfa, act.xo)]
    w4.linear(X0, pw, ws, Y[:0])
    w4.prep_act(X0, pw, act)
    w4.gemm_dual(act, 0, pw, Y[:0])
    w4.linear_noalloc(X0, pw, Y[:0])
    absmax = pw.act_scale.clone()
    w4.calib_observe(X0, absmax, reset=False)
    torch.cuda.synchronize()
    for a, b in zip(snap, (ws, Y, act.aq, act.sfa, act.xo)):
        assert torch.equal(a, b)
    assert torch.equal(absmax, pw.act_scale)
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"
    Y1 = _linear(X, pw, L.T, L.d_out)
    w4.linear(X, pw, ws, Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y1)


def test_gemm_matches_linear_and_is_deterministic():
    L = RAGGED
    X, W, pw = _calibrate(L)
    Y1 = _linear(X, pw, L.T, L.d_out)
    act = w4.alloc_act(L.T, pw)
    w4.prep_act(X, pw, act)
    Y2 = torch.empty_like(Y1)
    w4.gemm_dual(act, L.T, pw, Y2)
    Y3 = _linear(X, pw, L.T, L.d_out)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(Y1, Y3)


def test_linear_host_matches_device_path():
    L = RAGGED
    X, W, pw = _calibrate(L)
    Y = _linear(X, pw, L.T, L.d_out)
    Xh = X.cpu().pin_memory()
    Yh = torch.empty((L.T, L.d_out), dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty_like(X)
    Yd = torch.empty_like(Y)
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    w4.linear_host(Xh, pw, Xd, ws, Yd, Yh)
    torch.cuda.synchronize()
    assert torch.equal(Yh, Y.cpu())


def test_output_row_stride():
    L = RAGGED
    X, W, pw = _calibrate(L)
    Y = _linear(X, pw, L.T, L.d_out)
    big = torch.full((L.T, L.d_out + 32), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    w4.linear(X, pw, ws, big[:, :L.d_out])
    torch.cuda.synchronize()
    assert torch.equal(big[:, :L.d_out], Y)
    assert torch.all(big[:, L.d_out:] == 7.0)
