"""Failure detection on the GPU without a fault: a device pipeline wait that
runs out.  The failure-detection hook (w4a4_test_fault) shortens the wait
limit to 1 ms and makes the activation-prep producer issue no row copies, so
the consumers' waits on rows that never arrive run out: the kernel records
W4A4_ERR_TIMEOUT in the device error word and returns (no trap, no hang), and
once the hook is cleared the same calls give the same bits as before."""
import time

import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEVERR_TIMEOUT_PREP = 1 << 3

CASES = [
    # the block-per-lane prep kernel, and the 8-columns-per-lane one (rows past 15360)
    synth.Layer("fail_block", 300, 512, 384, 0.6, 8, 0, synth.X_UP, synth.W_UP, seed=31),
    synth.Layer("fail_wide", 200, 16384, 256, 0.6, 40, 0, synth.X_UP, synth.W_UP, seed=32),
]


@pytest.mark.parametrize("L", CASES, ids=lambda L: L.name)
def test_prep_wait_runs_out_and_the_context_recovers(L):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    ref = w4.alloc_act(L.T, pw)
    w4.prep_act(X, pw, ref)
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Y_ref = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    w4.linear(X, pw, ws, Y_ref)
    assert w4.last_error(clear=True)[0] == w4.OK

    act = w4.alloc_act(L.T, pw)
    w4.test_fault(w4.FAULT_PREP_SKIP_LOADS, 1_000_000)          # 1 ms waits, no row copies
    try:
        t0 = time.monotonic()
        w4.prep_act(X, pw, act)
        st, bits = w4.last_error(clear=True)                      # synchronises the stream
        took = time.monotonic() - t0
    finally:
        w4.test_fault(0, 0)
    assert st == w4.ERR_TIMEOUT, hex(bits)
    assert bits & DEVERR_TIMEOUT_PREP
    assert took < 5.0                                             # gave up, did not hang

    # the context is usable and the hook is gone: same bits as before the fault
    assert w4.last_error()[0] == w4.OK
    w4.prep_act(X, pw, act)
    Y = torch.empty_like(Y_ref)
    w4.linear(X, pw, ws, Y)
    assert w4.last_error()[0] == w4.OK
    assert torch.equal(act.aq, ref.aq) and torch.equal(act.xo, ref.xo)
    d = pw.dims
    np.testing.assert_array_equal(gu.sf_canonical(act.sfa, L.T, d.nblk, d.nblk),
                                  gu.sf_canonical(ref.sfa, L.T, d.nblk, d.nblk))
    assert torch.equal(Y, Y_ref)
