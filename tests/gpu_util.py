"""Helpers for the GPU parity tests: run the library on a layer and read its
device buffers back into the oracle's canonical host layouts."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import w4a4_oracle as orc


def to_np_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sf_canonical(flat: torch.Tensor, rows, nblk_lib: int, nblk_ref: int) -> np.ndarray:
    """Scale bytes in the MMA layout -> canonical [rows, nblk_lib] order (the
    blocks past nblk_ref are padding, returned for a zero check).  ``rows`` is
    a row count or an array of row indices."""
    buf = flat.cpu().numpy()
    r = (np.arange(rows) if np.isscalar(rows) else np.asarray(rows))[:, None]
    kb = np.arange(nblk_lib)[None, :]
    return buf[orc.mma_sf_offset(r, kb, nblk_lib)]


def check_tolerance(Y_gpu: np.ndarray, Y_ref: np.ndarray, what: str = ""):
    """|Y_gpu - Y_ref| <= 8e-3 |Y_ref| + 1e-3 rms(Y_ref), element by element."""
    rms = float(np.sqrt(np.mean(Y_ref.astype(np.float64) ** 2)))
    err = np.abs(Y_gpu.astype(np.float64) - Y_ref)
    bound = 8e-3 * np.abs(Y_ref) + 1e-3 * rms
    bad = err > bound
    ratio = float((err / bound).max()) if err.size else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, "
                           f"worst err/bound {ratio:.3f}")
    return ratio


def snr_db(Y: np.ndarray, Y_exact: np.ndarray) -> float:
    num = float((Y_exact ** 2).sum())
    den = float(((Y - Y_exact) ** 2).sum())
    return 10 * np.log10(num / den) if den > 0 else float("inf")


def oracle_calib_from_gpu(pw) -> dict:
    """Oracle O/J from the library's score, for the bit-exact downstream stages."""
    score = pw.score.cpu().numpy()
    O, J = orc.select_outliers(score, pw.k)
    return {"s": pw.s.cpu().numpy(), "inv_s": pw.inv_s.cpu().numpy(), "score": score, "O": O, "J": J}


def gen(layer: synth.Layer):
    X, W = synth.gen_layer(layer, "cuda")
    torch.cuda.synchronize()
    return X, W
