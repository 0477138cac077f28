"""The online path captured in a CUDA graph (the way a serving loop replays a
fixed-shape layer without launch overhead): `linear` (prep + GEMM) and the
fused FFN forward, replayed with new inputs copied into the captured buffers,
give the same bits as eager calls."""
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4
from w4a4_mxfp4_outlier_b200 import ffn
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

XS = synth.XSpec("student3", 0.3, 12, 8.0, 30.0)


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    return g


@pytest.mark.parametrize("T", [100, 600], ids=["single_cta", "pair"])
def test_linear_graph_replay(T):
    L = synth.Layer("graph", T, 1024, 768, 0.6, 16, 0, XS, synth.WSpec(0.02), seed=3)
    X, W = gu.gen(L)
    pw = w4.calibrate(X, W, L.alpha, L.k, L.layout)
    ws = torch.empty(w4.workspace_size(T, L.d_in, L.d_out, L.k), dtype=torch.uint8, device="cuda")
    Xg = X.clone()
    Yg = torch.empty((T, L.d_out), dtype=torch.bfloat16, device="cuda")
    g = _capture(lambda: w4.linear(Xg, pw, ws, Yg))
    X2, _ = gu.gen(L.with_(seed=11))
    for Xin in (X, X2, X):
        Xg.copy_(Xin)
        g.replay()
        Y = torch.empty_like(Yg)
        ws2 = torch.empty_like(ws)
        w4.linear(Xin, pw, ws2, Y)
        torch.cuda.synchronize()
        assert torch.equal(Yg.view(torch.int16), Y.view(torch.int16))
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)


def test_ffn_graph_replay():
    T, d_model, d_ff = 300, 512, 1376
    Lx = synth.Layer("ffn_graph", T, d_model, d_ff, 0.6, 8, 0, XS, synth.WSpec(0.02), seed=5)
    X, W_up = gu.gen(Lx)
    W_down = synth.gen_w(synth.WSpec(0.015), d_model, d_ff, seed=6, device="cuda")
    f = ffn.calibrate_ffn(X, W_up, W_down, 0.6, 8, 0.7, 19, 0)
    act_up, act_down = w4.alloc_act(T, f.up), w4.alloc_act(T, f.down)
    Xg = X.clone()
    Yg = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    g = _capture(lambda: ffn.forward(Xg, f, Yg, act_up, act_down))
    X2, _ = gu.gen(Lx.with_(seed=12))
    for Xin in (X2, X):
        Xg.copy_(Xin)
        g.replay()
        Y = torch.empty_like(Yg)
        ffn.forward(Xin, f, Y)
        torch.cuda.synchronize()
        assert torch.equal(Yg.view(torch.int16), Y.view(torch.int16))
    st, bits = w4.last_error()
    assert st == w4.OK, hex(bits)
