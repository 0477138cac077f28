"""Programmatic dependent launch: the calibration, finalisation, prep and GEMM
kernels may start their on-chip setup while the previous kernel in the
stream is finishing, and touch memory only after `griddepcontrol.wait`.

The whole chain -- calibration of X and W, finalisation, pack, prep, GEMM --
runs back to back on one stream with no synchronisation, reusing one
workspace and one output buffer from call to call, so that every kernel
overwrites what the previous call's kernels read.  It must give the same bits
as the same chain launched plainly (W4A4_NO_PDL=1; the switch is read once
per process, so that run is a child process)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth
import w4a4_mxfp4_outlier_b200 as w4

pytestmark = pytest.mark.gpu

LAYERS = [
    synth.FFN0.with_(name="pdl_up_T2048", T=2048, seed=41),
    synth.FFN2.with_(name="pdl_down_T2048", T=2048, seed=42),
    synth.Layer("pdl_ragged", 200, 136, 368, 0.6, 3, 1, synth.X_UP, synth.WSpec(0.02), seed=43),
]


def chain():
    """The chain for every layer; returns the bit patterns it produced."""
    data = []
    for L in LAYERS:
        X1, W = synth.gen_layer(L, "cuda")
        X2 = synth.gen_layer(L.with_(seed=L.seed + 100), "cuda")[0]
        data.append((L, X1, X2, W))
    torch.cuda.synchronize()
    outs = []
    for L, X1, X2, W in data:
        ws = torch.empty(w4.workspace_size(L.T, L.d_in, L.d_out, L.k), dtype=torch.uint8,
                         device="cuda")
        Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device="cuda")
        keep = []
        pw = w4.calibrate(X1, W, L.alpha, L.k, L.layout)
        for X in (X1, X2, X1):
            w4.linear(X, pw, ws, Y)               # same workspace and Y every time
            keep.append(Y.clone())
        pw2 = w4.calibrate([X2, X1], W, L.alpha, L.k, L.layout)
        w4.linear(X2, pw2, ws, Y)
        keep.append(Y.clone())
        keep += [pw.s, pw.inv_s, pw.wq, pw.sfb, pw2.act_scale, pw2.s]
        if L.k:
            keep += [pw.O, pw2.O]
        outs += keep
    torch.cuda.synchronize()
    st, bits = w4.last_error()
    assert st == w4.OK, f"device error word {bits:#x}"
    return [o.contiguous().view(torch.uint8).cpu().numpy() for o in outs]


_CHILD = """
import sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from tests import test_gpu_pdl as t
for i, o in enumerate(t.chain()):
    np.save(sys.argv[2] + f"/o{i}.npy", o)
"""


def test_dependent_launch_gives_the_bits_of_plain_launches(tmp_path):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, W4A4_NO_PDL="1")
    r = subprocess.run([sys.executable, "-c", _CHILD, root, str(tmp_path)], env=env, cwd=root,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    for rep in range(2):                          # the dependent-launch chain, twice
        outs = chain()
        for i, o in enumerate(outs):
            ref = np.load(tmp_path / f"o{i}.npy")
            assert np.array_equal(o, ref), f"output {i} differs (repetition {rep})"
