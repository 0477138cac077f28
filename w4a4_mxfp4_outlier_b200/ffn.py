"""The FFN pair (up projection, GELU, down projection) on the library.

The review quantises both FFN projections of the Wan2.2 DiT with the same
recipe (sec. 3.1, 3.5).  calibrate_ffn builds both packed layers; with the
up layer's packed rows reordered into the down layer's compacted input order
(w4a4_ffn_link / w4a4_permute_packed_rows), forward() runs

    prep_act(X) -> gemm_dual_act (up; its epilogue applies GELU and the down
    layer's activation prep) -> gemm_dual (down)

so the up layer's bf16 output never goes to memory.  forward_unfused() is
the same computation with the up output materialised (gemm_dual, gelu_bf16,
prep_act): the two give bit-identical Y.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import (PackedWeight, SF_32x1_KMAJOR, _check, _ffn_link, _gelu_bf16, _gemm_dual_act, _nz,
               _permute_packed_rows, _ptr, _stream, ActBuffers, alloc_act, alloc_packed, calib_finalize,
               calib_observe, calibrate, gemm_dual, linear, pack_weight, prep_act, workspace_size)


@dataclass
class PackedFFN:
    up: PackedWeight            # output channels in the down layer's compacted order
    down: PackedWeight
    perm: torch.Tensor          # int32 [d_ff]: up output column c is hidden channel perm[c]
    inv_s_perm: torch.Tensor    # float32 [d_ff]: down inv_s in that order
    up_plain: PackedWeight      # the up layer in its natural channel order (unfused path)


def gelu_bf16(Y: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    X = torch.empty_like(Y) if out is None else out
    _check(_gelu_bf16(_ptr(Y), Y.shape[0], Y.shape[1], Y.stride(0), _ptr(X), X.stride(0),
                      _stream(stream)), "gelu_bf16")
    return X


def calibrate_ffn(X_batches, W_up: torch.Tensor, W_down: torch.Tensor, alpha_up: float, k_up: int,
                  alpha_down: float, k_down: int, layout: int = SF_32x1_KMAJOR,
                  stream=None) -> PackedFFN:
    """Calibrates and packs both projections.  The down layer is calibrated on
    X_down = bf16(gelu(Y_up)) of every calibration batch."""
    batches = [X_batches] if isinstance(X_batches, torch.Tensor) else list(X_batches)
    d_ff, d_model = W_up.shape
    dev = W_up.device
    up_plain = calibrate(batches, W_up, alpha_up, k_up, layout, stream=stream)
    down = alloc_packed(d_ff, W_down.shape[0], k_down, layout, dev)
    for i, Xb in enumerate(batches):
        T = Xb.shape[0]
        ws = torch.empty(workspace_size(T, d_model, d_ff, k_up), dtype=torch.uint8, device=dev)
        Y = torch.empty((T, d_ff), dtype=torch.bfloat16, device=dev)
        linear(Xb, up_plain, ws, Y, stream=stream)
        calib_observe(gelu_bf16(Y, stream=stream), down.act_scale, reset=(i == 0), stream=stream)
    calib_observe(W_down, down.w_scale, reset=True, stream=stream)
    calib_finalize(down.act_scale, down.w_scale, alpha_down, k_down, down.s, down.inv_s, down.score,
                   down.O if k_down else None, down.jmap if k_down < d_ff else None, stream=stream)
    pack_weight(W_down, down, stream=stream)
    perm = torch.empty(d_ff, dtype=torch.int32, device=dev)
    inv_s_perm = torch.empty(d_ff, dtype=torch.float32, device=dev)
    _check(_ffn_link(ctypes.byref(down.c), _ptr(perm), _ptr(inv_s_perm), _stream(stream)),
           "ffn_link")
    up = alloc_packed(d_model, d_ff, k_up, layout, dev)
    # the input-side calibration of the up layer is unchanged by permuting its outputs
    up.s, up.inv_s, up.score, up.O, up.jmap = (up_plain.s, up_plain.inv_s, up_plain.score,
                                               up_plain.O, up_plain.jmap)
    up.act_scale, up.w_scale = up_plain.act_scale, up_plain.w_scale
    # reorder the natural pack (not a pack of the reordered W): every output
    # channel keeps its quantisation, 32x32 tiles included, so the fused and
    # unfused FFN compute the same function
    _check(_permute_packed_rows(ctypes.byref(up_plain.c), _ptr(perm), ctypes.byref(up.c),
                                _stream(stream)), "permute_packed_rows")
    return PackedFFN(up, down, perm, inv_s_perm, up_plain)


def gemm_dual_act(act_up: ActBuffers, T: int, f: PackedFFN, act_down: ActBuffers, stream=None):
    _check(_gemm_dual_act(_nz(act_up.aq), _nz(act_up.sfa), _nz(act_up.xo), T, ctypes.byref(f.up.c),
                          ctypes.byref(f.down.c), _ptr(f.inv_s_perm), _nz(act_down.aq),
                          _nz(act_down.sfa), _nz(act_down.xo), _stream(stream)), "gemm_dual_act")


def forward(X: torch.Tensor, f: PackedFFN, Y: torch.Tensor, act_up: ActBuffers | None = None,
            act_down: ActBuffers | None = None, stream=None):
    T = X.shape[0]
    act_up = act_up or alloc_act(T, f.up)
    act_down = act_down or alloc_act(T, f.down)
    prep_act(X, f.up, act_up, stream=stream)
    gemm_dual_act(act_up, T, f, act_down, stream=stream)
    gemm_dual(act_down, T, f.down, Y, stream=stream)
    return act_down


def forward_unfused(X: torch.Tensor, f: PackedFFN, Y: torch.Tensor, stream=None) -> torch.Tensor:
    """Returns the materialised hidden X_down; Y gets the down output."""
    T = X.shape[0]
    d_ff = f.up.d_out
    ws = torch.empty(workspace_size(T, X.shape[1], d_ff, f.up.k), dtype=torch.uint8, device=X.device)
    Yu = torch.empty((T, d_ff), dtype=torch.bfloat16, device=X.device)
    linear(X, f.up_plain, ws, Yu, stream=stream)
    H = gelu_bf16(Yu, stream=stream)
    ws2 = torch.empty(workspace_size(T, d_ff, f.down.d_out, f.down.k), dtype=torch.uint8,
                      device=X.device)
    linear(H, f.down, ws2, Y, stream=stream)
    return H
