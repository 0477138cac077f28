"""w4a4_linear_noalloc, the online layer on the library's fixed scratch array
(no allocation, no workspace argument), called through the C ABI and checked
against w4a4_linear with a caller workspace on the same inputs: bit for bit
(both run the same deterministic kernels), and the result against the
oracle's float64 product within the tolerance of the other parity tests.

The file is collected last on purpose: it must pass after every other GPU test
has run (whatever they left on the device) as well as alone.  The calls run
back to back on one stream, so each one starts from whatever the previous call
left in the shared scratch."""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# a ragged tail in every dimension, a 32x32-tile weight layout with k = 0 ... 256
RAGGED = synth.Layer("noalloc_ragged", 200, 136, 368, 0.6, 3, 0,
                     synth.XSpec("student3", 0.3, 4, 8.0, 30.0), synth.WSpec(0.02), seed=11)
MID = synth.Layer("noalloc_mid", 1000, 5120, 1024, 0.7, 256, 1, synth.X_UP, synth.W_UP, seed=12)
NO_OUTLIERS = synth.Layer("noalloc_k0", 130, 512, 272, 0.5, 0, 0, synth.X_TINY, synth.WSpec(0.02),
                          seed=13)
LARGEST = synth.Layer("noalloc_near_limit", 11000, 5120, 1024, 0.6, 32, 0, synth.X_UP, synth.W_UP,
                      seed=14)


def _prepare(L):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Y_ref = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, pw, ws, Y_ref)
    return X, pw, Y_ref


def _noalloc(X, pw, L):
    Y = torch.full((L.T, L.d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    w4.linear_noalloc(X, pw, Y)
    return Y


def test_noalloc_matches_linear_on_consecutive_calls():
    layers = [LARGEST, RAGGED, MID, NO_OUTLIERS]
    assert w4.workspace_size(LARGEST.T, LARGEST.d_in, LARGEST.d_out, LARGEST.k) \
        <= w4.NOALLOC_SCRATCH_BYTES
    prepared = [(L, *_prepare(L)) for L in layers]
    # every layer twice in a row, then the whole sequence again in reverse, so
    # each call finds the scratch left by a different earlier problem
    order = [p for p in prepared for _ in range(2)] + prepared[::-1]
    for L, X, pw, Y_ref in order:
        Y = _noalloc(X, pw, L)
        st, bits = w4.last_error()
        assert st == w4.OK, f"{L.name}: device error word {bits:#x}"
        # the same two deterministic kernels on the same inputs: any difference,
        # however small, would be scratch left over from an earlier call
        assert torch.equal(Y, Y_ref), f"{L.name}: no-alloc output differs from w4a4_linear"
    # and the shared result against the oracle's float64 product (sampled rows)
    for L, X, pw, Y_ref in prepared:
        _oracle_check(L, X, pw, Y_ref)


def _oracle_check(L, X, pw, Y, nrows=64):
    rows = np.unique(np.random.default_rng(5).integers(0, L.T, nrows))
    rows = np.union1d(rows, [0, L.T - 1])
    c = gu.oracle_calib_from_gpu(pw)
    Xs = gu.to_np_f32(X[torch.from_numpy(rows).cuda()])
    pwr = orc.pack_weight(gu.to_np_f32(gu.gen(L)[1]), c["s"], c["O"], c["J"], L.layout)
    pa = orc.prep_activation(Xs, c["inv_s"], c["O"], c["J"])
    Y_ref = orc.dual_branch_product(pa["aq"], pa["sfa"], pa["xo"], pwr["wq"], pwr["sfb"],
                                    pwr["w_hp"])
    gu.check_tolerance(gu.to_np_f32(Y[torch.from_numpy(rows).cuda()]).astype(np.float64), Y_ref,
                       f"{L.name} against the oracle")


def test_noalloc_rejects_problems_beyond_the_scratch():
    L = LARGEST.with_(name="noalloc_too_big", T=12100)
    assert w4.workspace_size(L.T, L.d_in, L.d_out, L.k) > w4.NOALLOC_SCRATCH_BYTES
    X, W = gu.gen(LARGEST)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    Xbig = torch.zeros((L.T, L.d_in), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A4Error) as e:
        w4.linear_noalloc(Xbig, pw, Y)
    assert e.value.status == w4.ERR_SCRATCH_LIMIT
    # the rejected call enqueued nothing and the entry point still works
    st, _ = w4.last_error()
    assert st == w4.OK
    Y_ref = torch.empty((LARGEST.T, LARGEST.d_out), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(w4.workspace_size(LARGEST.T, L.d_in, L.d_out, L.k), dtype=torch.uint8,
                     device="cuda")
    w4.linear(X, pw, ws, Y_ref)
    assert torch.equal(_noalloc(X, pw, LARGEST), Y_ref), "after rejection"
