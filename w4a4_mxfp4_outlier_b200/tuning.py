"""Layer-wise choice of alpha, k and the weight-scale layout.

The review ("W4A4 Quantization for Inference on Wan2.2-I2V-A14B", sec. 4
table "Layer-wise alpha and k", sec. 6) proposes different alpha and k for
shallow and deep layers as the next step, without a procedure.  The plainest
one, used here: run the whole quantised layer for every candidate on
calibration activations and keep the candidate with the smallest relative
Frobenius error ||Y - X W^T|| / ||X W^T||, preferring the smaller k (the
high-precision budget) on ties, then the candidate listed first (layouts,
then k, then alpha, in the order given).

Every candidate runs through the library: calib_observe once (the absmax
statistics do not depend on alpha or k), then calib_finalize, pack_weight,
linear and error_sums per candidate.  The reference product X W^T is a plain
float32 cuBLAS GEMM (torch.matmul): an evaluation-only reference for scoring
candidates, not a step of the quantised layer.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import (SF_32x1_KMAJOR, _check, _error_sums, _stream, alloc_packed, calib_finalize,
               calib_observe, linear, pack_weight, workspace_size)


@dataclass
class SearchResult:
    best: tuple                                  # (alpha, k, layout)
    errors: dict = field(default_factory=dict)   # (alpha, k, layout) -> relative error


def relative_error(Y: torch.Tensor, Yref: torch.Tensor, stream=None) -> float:
    """sqrt(sum (Y - Yref)^2 / sum Yref^2) with Y bf16 and Yref float32 on the device."""
    sums = torch.empty(2, dtype=torch.float64, device=Y.device)
    _check(_error_sums(Y.data_ptr(), Y.stride(0), Yref.data_ptr(), Yref.stride(0), Y.shape[0],
                       Y.shape[1], sums.data_ptr(), _stream(stream)), "error_sums")
    num, den = sums.tolist()
    return (num / den) ** 0.5 if den > 0 else 0.0


def search_layer(X_calib, W: torch.Tensor, alphas, ks, layouts=(SF_32x1_KMAJOR,), X_eval=None,
                 stream=None) -> SearchResult:
    """Scores every (alpha, k, layout) on X_eval (default: the first
    calibration batch) and returns the best with the whole table."""
    batches = [X_calib] if isinstance(X_calib, torch.Tensor) else list(X_calib)
    Xe = batches[0] if X_eval is None else X_eval
    d_out, d_in = W.shape
    act = torch.empty(d_in, dtype=torch.float32, device=W.device)
    wsc = torch.empty(d_in, dtype=torch.float32, device=W.device)
    for i, Xb in enumerate(batches):
        calib_observe(Xb, act, reset=(i == 0), stream=stream)
    calib_observe(W, wsc, reset=True, stream=stream)
    Yref = torch.matmul(Xe.float(), W.float().t())
    T = Xe.shape[0]
    Y = torch.empty((T, d_out), dtype=torch.bfloat16, device=W.device)
    result = SearchResult(best=None)
    for layout in layouts:
        for k in ks:
            ws = torch.empty(workspace_size(T, d_in, d_out, k), dtype=torch.uint8, device=W.device)
            for alpha in alphas:
                pw = alloc_packed(d_in, d_out, k, layout, W.device)
                calib_finalize(act, wsc, alpha, k, pw.s, pw.inv_s, pw.score,
                               pw.O if k else None, pw.jmap if k < d_in else None, stream=stream)
                pack_weight(W, pw, stream=stream)
                linear(Xe, pw, ws, Y, stream=stream)
                result.errors[(alpha, k, layout)] = relative_error(Y, Yref, stream)
    result.best = min(result.errors, key=lambda c: (result.errors[c], c[1]))
    return result
