"""Packed-weight checkpoints on the GPU: save -> load reproduces every
buffer byte for byte and the loaded layer computes the same Y."""
import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

LAYERS = [synth.TINY,
          synth.Layer("ckpt_ragged_32x32", 200, 136, 368, 0.6, 11, 1,
                      synth.XSpec("student3", 0.3, 4, 8.0, 30.0), synth.WSpec(0.02), seed=3),
          synth.TINY.with_(name="ckpt_k0_128x1", k=0, layout=2)]


@pytest.mark.parametrize("L", LAYERS, ids=lambda L: L.name)
def test_checkpoint_roundtrip(L, tmp_path):
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    path = str(tmp_path / "layer.w4a4")
    w4.save_packed(pw, path)
    pl = w4.load_packed(path)
    assert (pl.d_in, pl.d_out, pl.k, pl.layout) == (L.d_in, L.d_out, L.k, L.layout)
    for name in ("wq", "sfb", "w_hp", "s", "inv_s", "O", "jmap"):
        a, b = getattr(pw, name), getattr(pl, name)
        assert torch.equal(a.view(torch.uint8) if a.numel() else a,
                           b.view(torch.uint8) if b.numel() else b), name
    ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Y0 = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
    Y1 = torch.empty_like(Y0)
    w4.linear(X, pw, ws, Y0)
    w4.linear(X, pl, ws, Y1)
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))


def test_checkpoint_rejects_corruption():
    L = synth.TINY
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    img = bytearray(w4.packed_to_bytes(pw))
    img[len(img) // 2] ^= 0x40                       # one payload bit
    with pytest.raises(w4.W4A4Error) as e:
        w4.packed_from_bytes(bytes(img))
    assert e.value.status == w4.ERR_BAD_IMAGE
    # a record of other dims refuses the image
    good = w4.packed_to_bytes(pw)
    other = w4.alloc_packed(L.d_in, L.d_out, L.k + 1, L.layout)
    buf = torch.frombuffer(bytearray(good), dtype=torch.uint8)
    import ctypes
    st = w4._packed_load(buf.data_ptr(), buf.numel(), ctypes.byref(other.c), other.s.data_ptr(), None)
    assert st == w4.ERR_INVALID_ARG
