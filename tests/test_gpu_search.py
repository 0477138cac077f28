"""Layer-wise (alpha, k, layout) search on the GPU against the oracle's
search on the same inputs.

Per candidate, the GPU error (Y from the library against a float32 X W^T)
and the oracle's (its float64 Y against the exact float64 X W^T) differ only
by the GPU-vs-oracle Y difference, at most 8e-3 |Y| + 1e-3 rms(Y) per element
(the parity bound), so by at most about 0.01 absolute on errors of 0.07-0.2.
Several candidates sit within that of each other, so the GPU's choice is
checked to be near-optimal by the oracle's table rather than identical."""
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from w4a4_mxfp4_outlier_b200 import tuning
from oracle import w4a4_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

ALPHAS = (0.3, 0.5, 0.7)
KS = (0, 4, 8, 16)
LAYOUTS = (w4.SF_32x1_KMAJOR, w4.SF_32x32_TILE, w4.SF_128x1_KMAJOR)


def test_search_matches_oracle():
    L = synth.TINY
    X, W = gu.gen(L)
    res = tuning.search_layer(X, W, ALPHAS, KS, LAYOUTS)
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)
    best_o, err_o = orc.search_layer(gu.to_np_f32(X), gu.to_np_f32(W), ALPHAS, KS, LAYOUTS)
    assert set(res.errors) == set(err_o)
    for c, e in res.errors.items():
        assert abs(e - err_o[c]) <= 0.01 + 0.02 * err_o[c], (c, e, err_o[c])
    # the GPU's choice is within the comparison noise of the oracle's optimum
    assert err_o[res.best] <= err_o[best_o] + 0.01 + 0.02 * err_o[best_o]
    # protecting the 8 planted channels is what matters most on this layer
    assert res.best[1] >= 8


def test_relative_error_kernel():
    torch.manual_seed(0)
    R = torch.randn(300, 272, device="cuda")
    Y = (R + 0.01 * torch.randn_like(R)).to(torch.bfloat16)
    e = tuning.relative_error(Y, R)
    ref = ((Y.double() - R.double()).pow(2).sum() / R.double().pow(2).sum()).sqrt().item()
    assert abs(e - ref) <= 1e-9 * max(1.0, ref)
    assert tuning.relative_error(R.to(torch.bfloat16)[:0], R[:0]) == 0.0


def test_search_hand_worked_case():
    """The hand-worked case of tests/golden/search_layer_hand.txt on the GPU:
    every quantised product there is exact in bf16 and the reference product
    is exact in float32, so the library's errors are the hand values."""
    from tests import search_hand_case as hc
    X, W = hc.inputs()
    Xg = torch.from_numpy(X).to(torch.bfloat16).cuda()
    Wg = torch.from_numpy(W).to(torch.bfloat16).cuda()
    res = tuning.search_layer(Xg, Wg, hc.ALPHAS, hc.KS)
    assert w4.last_error()[0] == w4.OK
    table, best = hc.expected()
    assert set(res.errors) == set(table)
    for c, e in table.items():
        assert abs(res.errors[c] - e) <= 1e-12, (c, res.errors[c], e)
    assert res.best == best
