"""Planted mistakes in the CPU oracle, for showing that its pins catch them.

A pytest plugin: run as ``pytest -p tests.oracle_mutants`` with
W4A4_ORACLE_MUTANT=<name>, it replaces one oracle function by a plausibly
wrong variant before any test runs (on the CPU, in that process only).
tests/test_oracle_mutants.py runs the oracle's pin files once per mutant
and requires each run to fail.  Each mutant is a mistake someone could make
when writing the method down: a rounding rule, an exponent, an index order,
a dropped term, an operand used the wrong way round.
"""
import os

import numpy as np

from oracle import w4a4_oracle as orc

_orig = {name: getattr(orc, name) for name in (
    "e2m1_codes", "mx_shared_exponent", "pack_nibbles", "unpack_nibbles",
    "smoothing_factors", "outlier_scores", "select_outliers", "fold_weight",
    "dual_branch_product", "pack_weight", "f32_to_bf16_bits", "gelu_bf16",
    "col_absmax")}


def _e2m1_ties_away(q):
    """Ties to the larger magnitude instead of to the even code."""
    a = np.minimum(np.abs(np.asarray(q, dtype=np.float64)), orc.E2M1_GRID[-1])
    d = np.abs(a[..., None] - orc.E2M1_GRID)
    cand = d == d.min(axis=-1, keepdims=True)
    pick = 7 - np.argmax(cand[..., ::-1], axis=-1)
    sign = np.signbit(np.asarray(q, dtype=np.float32)).astype(np.int64)
    return (pick | (sign << 3)).astype(np.uint8)


def _e2m1_unsigned_zero(q):
    """-0 (and values rounding to 0) lose their sign bit."""
    c = _orig["e2m1_codes"](q)
    return np.where((c & 7) == 0, 0, c).astype(np.uint8)


def _exponent_minus_1(amax):
    """Shared exponent floor(log2 amax) - 1 (E2M1's emax taken as 1)."""
    e = _orig["mx_shared_exponent"](amax)
    return np.where(np.asarray(amax) == 0.0, e, np.clip(e + 1, -127, 127))


def _pack_high_first(codes):
    """Element 2i in the high nibble (and read back the same way)."""
    c = codes.astype(np.uint8)
    return (c[..., 1::2] | (c[..., 0::2] << 4)).astype(np.uint8)


def _unpack_high_first(b):
    b = b.astype(np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = b >> 4
    out[..., 1::2] = b & 0xF
    return out


def _alpha_swapped(act_scale, w_scale, alpha):
    """s = act^(1-alpha) / w^alpha: the two exponents exchanged."""
    return _orig["smoothing_factors"](act_scale, w_scale, 1.0 - alpha)


def _s_for_inv_s(act_scale, w_scale, alpha):
    """The online path multiplies by s instead of 1/s."""
    s, _ = _orig["smoothing_factors"](act_scale, w_scale, alpha)
    return s, s.copy()


def _score_unsmoothed(X, inv_s):
    """Outlier score on the raw activations (splitting before smoothing)."""
    return np.max(np.abs(X.astype(np.float32)), axis=0).astype(np.float32)


def _topk_ties_high(score, k):
    """Equal scores go to the higher column index."""
    d = score.shape[0]
    idx = np.arange(d)
    order = np.lexsort((-idx, -score.astype(np.float64)))
    return np.sort(order[:k]).astype(np.int32), np.sort(order[k:]).astype(np.int32)


def _fold_divides(W, s):
    """The weights divided by s instead of multiplied."""
    return W / s[None, :]


def _drop_outlier_branch(aq, sfa, xo, wq, sfb, w_hp):
    """Y without the X_O W_hp term."""
    return orc.dequant_mxfp4(aq, sfa) @ orc.dequant_mxfp4(wq, sfb).T


def _tiles_as_rows(W, s, O, J, layout=orc.LAYOUT_32x1, row_chunk=512):
    """32x32 tiles packed with one scale per 32x1 block."""
    if layout == orc.LAYOUT_32x32:
        layout = orc.LAYOUT_32x1
    return _orig["pack_weight"](W, s, O, J, layout, row_chunk)


def _bf16_truncate(x):
    """float32 -> bfloat16 by truncation instead of round-to-nearest-even."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    return (b >> 16).astype(np.uint16)


def _gelu_erf(y):
    """GELU in its erf form (the pages' FFN uses the tanh form)."""
    from scipy.special import erf
    yv = np.asarray(y, dtype=np.float64)
    return orc.f64_to_bf16_bits(0.5 * yv * (1.0 + erf(yv / np.sqrt(2.0))))


def _absmax_signed(A, running=None):
    """Column max of the values instead of their magnitudes."""
    m = np.max(A.astype(np.float32), axis=0) if A.shape[0] else np.zeros(A.shape[1], np.float32)
    if running is not None:
        m = np.maximum(m, running)
    return m.astype(np.float32)


MUTANTS = {
    "e2m1_ties_away": {"e2m1_codes": _e2m1_ties_away},
    "e2m1_unsigned_zero": {"e2m1_codes": _e2m1_unsigned_zero},
    "exponent_minus_1": {"mx_shared_exponent": _exponent_minus_1},
    "nibbles_high_first": {"pack_nibbles": _pack_high_first, "unpack_nibbles": _unpack_high_first},
    "alpha_swapped": {"smoothing_factors": _alpha_swapped},
    "s_for_inv_s": {"smoothing_factors": _s_for_inv_s},
    "score_unsmoothed": {"outlier_scores": _score_unsmoothed},
    "topk_ties_high": {"select_outliers": _topk_ties_high},
    "fold_divides": {"fold_weight": _fold_divides},
    "drop_outlier_branch": {"dual_branch_product": _drop_outlier_branch},
    "tiles_as_rows": {"pack_weight": _tiles_as_rows},
    "bf16_truncate": {"f32_to_bf16_bits": _bf16_truncate},
    "gelu_erf": {"gelu_bf16": _gelu_erf},
    "absmax_signed": {"col_absmax": _absmax_signed},
}


def pytest_configure(config):
    name = os.environ.get("W4A4_ORACLE_MUTANT", "")
    if not name:
        return
    if name != "none":
        for attr, fn in MUTANTS[name].items():
            setattr(orc, attr, fn)
