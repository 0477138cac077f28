"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every symbol include/w4a4.h declares, and validates arguments before any
launch (invalid calls return an error status and enqueue nothing)."""
import ctypes
import os
import re

import pytest

import w4a4_mxfp4_outlier_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "w4a4.h")).read()
    return sorted(set(re.findall(r"\b(w4a4_[a-z_0-9]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(w4.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(w4.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings():
    assert w4.abi_version() == 1
    assert w4.status_string(w4.OK) == "ok"
    assert "timed out" in w4.status_string(w4.ERR_TIMEOUT)


def test_dims():
    d = w4.get_dims(5120, 13824, 32)
    assert (d.kj, d.kj_pad, d.nblk, d.k_pad, d.sfb_rows) == (5088, 5120, 160, 32, 13824)
    d = w4.get_dims(13824, 5120, 64)
    assert (d.kj, d.kj_pad, d.nblk, d.k_pad) == (13760, 13824, 432, 64)
    d = w4.get_dims(512, 512, 8)
    assert (d.kj_pad, d.k_pad, d.sfb_rows) == (512, 16, 512)
    d = w4.get_dims(5120, 13824, 0)
    assert (d.kj_pad, d.k_pad) == (5120, 0)
    d = w4.get_dims(64, 48, 64)
    assert (d.kj, d.kj_pad, d.nblk, d.sfb_rows) == (0, 0, 0, 256)


def test_sizes():
    b = w4.weight_sizes(5120, 13824, 32)
    assert (b.wq, b.sfb, b.w_hp) == (13824 * 2560, 13824 * 160, 13824 * 32 * 2)
    n = w4.workspace_size(4096, 5120, 13824, 32)
    assert n == 4096 * 2560 + 4096 * 160 + 4096 * 32 * 2
    assert w4.workspace_size(100, 512, 512, 8) >= 100 * 256 + 128 * 16 + 100 * 16 * 2


@pytest.mark.parametrize("args,status", [
    ((0, 16, 0), w4.ERR_INVALID_ARG),
    ((64, 16, 65), w4.ERR_INVALID_ARG),
    ((60, 16, 0), w4.ERR_UNSUPPORTED_SHAPE),      # d_in % 8
    ((64, 24, 0), w4.ERR_UNSUPPORTED_SHAPE),      # d_out % 16
    ((70000, 16, 0), w4.ERR_UNSUPPORTED_SHAPE),   # d_in > 65535
])
def test_weight_sizes_rejects(args, status):
    with pytest.raises(w4.W4A4Error) as e:
        w4.weight_sizes(*args)
    assert e.value.status == status


def _raw_pw(d_in=64, d_out=32, k=4, layout=0, fake=0x1000):
    return w4.PackedWeightC(d_in, d_out, k, layout, 0, fake, fake, fake, fake, fake, fake)


def test_calls_validate_before_launch():
    # Pointers here are never dereferenced: every call must fail validation.
    pw = _raw_pw()
    st = w4._prep_act(0x1000, 8, 63, ctypes.byref(pw), 0x1000, 0x1000, 0x1000, None)  # ldx < d_in
    assert st == w4.ERR_INVALID_ARG
    st = w4._prep_act(0x1000, 8, 68, ctypes.byref(pw), 0x1000, 0x1000, 0x1000, None)  # ldx % 8
    assert st == w4.ERR_UNSUPPORTED_SHAPE
    st = w4._prep_act(0x1001, 8, 64, ctypes.byref(pw), 0x1000, 0x1000, 0x1000, None)  # misaligned X
    assert st == w4.ERR_UNSUPPORTED_SHAPE
    st = w4._gemm_dual(0x1000, 0x1000, 0x1000, 8, ctypes.byref(pw), 0x1000, 31, None)  # ldy < d_out
    assert st == w4.ERR_INVALID_ARG
    st = w4._gemm_dual(0x1000, 0x1000, None, 8, ctypes.byref(pw), 0x1000, 32, None)  # xo missing, k>0
    assert st == w4.ERR_INVALID_ARG
    bad = _raw_pw(layout=7)
    assert w4._gemm_dual(0x1000, 0x1000, 0x1000, 8, ctypes.byref(bad), 0x1000, 32, None) == w4.ERR_INVALID_ARG
    st = w4._linear(0x1000, 8, 64, ctypes.byref(pw), 0x1000, 16, 0x1000, 32, None)  # workspace too small
    assert st == w4.ERR_INVALID_ARG
    assert w4._prep_act(0x1000, 8, 64, None, 0x1000, 0x1000, 0x1000, None) == w4.ERR_INVALID_ARG
    # T == 0 is a valid no-op that launches nothing
    assert w4._prep_act(None, 0, 64, ctypes.byref(pw), None, None, None, None) == w4.OK
    assert w4._gemm_dual(None, None, None, 0, ctypes.byref(pw), None, 32, None) == w4.OK


def test_ffn_calls_validate_before_launch():
    # Pointers here are never dereferenced: every call returns before any CUDA work.
    f = 0x1000
    pw = _raw_pw()                                  # 64 -> 32, k = 4
    nxt = _raw_pw(d_in=32, d_out=64, k=4, fake=0x2000)
    # GELU: row strides below the width, missing buffers, negative T; empty is a no-op
    assert w4._gelu_bf16(f, 8, 64, 63, f, 64, None) == w4.ERR_INVALID_ARG
    assert w4._gelu_bf16(f, 8, 64, 64, f, 63, None) == w4.ERR_INVALID_ARG
    assert w4._gelu_bf16(None, 8, 64, 64, f, 64, None) == w4.ERR_INVALID_ARG
    assert w4._gelu_bf16(f, -1, 64, 64, f, 64, None) == w4.ERR_INVALID_ARG
    assert w4._gelu_bf16(None, 0, 64, 64, None, 64, None) == w4.OK
    # channel order of the next layer: a valid packed layer and both outputs
    assert w4._ffn_link(None, f, f, None) == w4.ERR_INVALID_ARG
    assert w4._ffn_link(ctypes.byref(nxt), None, f, None) == w4.ERR_INVALID_ARG
    assert w4._ffn_link(ctypes.byref(_raw_pw(layout=7)), f, f, None) == w4.ERR_INVALID_ARG
    # packing permuted rows: the same checks as the plain pack, plus the row map
    assert w4._pack_weight_rows(f, 63, f, f, ctypes.byref(pw), None) == w4.ERR_INVALID_ARG
    assert w4._pack_weight_rows(f, 68, f, f, ctypes.byref(pw), None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._pack_weight_rows(f + 2, 64, f, f, ctypes.byref(pw), None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._pack_weight_rows(f, 64, f, None, ctypes.byref(pw), None) == w4.ERR_INVALID_ARG
    # permuting a packed layer: same shape and layout, a row map, never in place
    other = _raw_pw(fake=0x3000)
    assert w4._permute_packed_rows(ctypes.byref(pw), f, ctypes.byref(_raw_pw(d_out=48, fake=0x3000)),
                                   None) == w4.ERR_INVALID_ARG
    assert w4._permute_packed_rows(ctypes.byref(pw), f, ctypes.byref(_raw_pw(layout=1, fake=0x3000)),
                                   None) == w4.ERR_INVALID_ARG
    assert w4._permute_packed_rows(ctypes.byref(pw), None, ctypes.byref(other), None) == w4.ERR_INVALID_ARG
    assert w4._permute_packed_rows(ctypes.byref(pw), f, ctypes.byref(_raw_pw()), None) == w4.ERR_INVALID_ARG
    # the fused epilogue: the next layer's d_in is this layer's d_out, its
    # column order's inv_s is given, its buffers are there and 16-byte aligned
    act = lambda T=8, nx=nxt, inv=f, aqn=f + 0x100: w4._gemm_dual_act(
        f, f, f, T, ctypes.byref(pw), ctypes.byref(nx), inv, aqn, f + 0x200, f + 0x300, None)
    assert act(nx=_raw_pw(d_in=48, d_out=64, fake=0x2000)) == w4.ERR_INVALID_ARG
    assert act(inv=None) == w4.ERR_INVALID_ARG
    assert act(T=-1) == w4.ERR_INVALID_ARG
    assert act(aqn=None) == w4.ERR_INVALID_ARG
    assert act(aqn=f + 0x101) == w4.ERR_UNSUPPORTED_SHAPE
    assert act(T=0) == w4.OK


def test_pack_host_and_metric_calls_validate_before_launch():
    # Pointers here are never dereferenced: every call returns before any CUDA work.
    f = 0x1000
    pw = _raw_pw()                                  # 64 -> 32, k = 4
    # weight pack: row stride, alignment, missing W or s, a malformed record
    assert w4._pack_weight(f, 63, f, ctypes.byref(pw), None) == w4.ERR_INVALID_ARG
    assert w4._pack_weight(f, 68, f, ctypes.byref(pw), None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._pack_weight(f + 8, 64, f, ctypes.byref(pw), None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._pack_weight(None, 64, f, ctypes.byref(pw), None) == w4.ERR_INVALID_ARG
    assert w4._pack_weight(f, 64, None, ctypes.byref(pw), None) == w4.ERR_INVALID_ARG
    no_inv = _raw_pw()
    no_inv.inv_s = None
    assert w4._pack_weight(f, 64, f, ctypes.byref(no_inv), None) == w4.ERR_INVALID_ARG
    # the host-buffer layer: every buffer, a big enough workspace; T = 0 is a no-op
    ws = w4.workspace_size(8, 64, 32, 4)
    assert w4._linear_host(f, -1, ctypes.byref(pw), f, f, ws, f, f, None) == w4.ERR_INVALID_ARG
    assert w4._linear_host(None, 8, ctypes.byref(pw), f, f, ws, f, f, None) == w4.ERR_INVALID_ARG
    assert w4._linear_host(f, 8, ctypes.byref(pw), f, f, ws, f, None, None) == w4.ERR_INVALID_ARG
    assert w4._linear_host(f, 8, ctypes.byref(pw), f, f, ws - 1, f, f, None) == w4.ERR_INVALID_ARG
    assert w4._linear_host(f, 0, ctypes.byref(pw), None, None, 0, None, None, None) == w4.OK
    # the error-sum reduction used by the layer search
    assert w4._error_sums(f, 31, f, 32, 8, 32, f, None) == w4.ERR_INVALID_ARG
    assert w4._error_sums(f, 32, f, 31, 8, 32, f, None) == w4.ERR_INVALID_ARG
    assert w4._error_sums(f, 32, f, 32, 8, 32, None, None) == w4.ERR_INVALID_ARG
    assert w4._error_sums(None, 32, f, 32, 8, 32, f, None) == w4.ERR_INVALID_ARG


def test_calib_validation():
    assert w4._calib_observe(0x1000, 4, 8, 4, 0x1000, 1, None) == w4.ERR_INVALID_ARG      # lda < cols
    assert w4._calib_observe(0x1000, 4, 12, 12, 0x1000, 1, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._calib_observe(None, 4, 8, 8, 0x1000, 1, None) == w4.ERR_INVALID_ARG
    f = 0x1000
    # the one-launch layer form: X [T, d_in] and W [d_out, d_in]
    lay = w4._calib_observe_layer
    assert lay(f, 4, 8, f, 4, 8, 8, f, f, 1, None) == w4.ERR_INVALID_ARG          # outputs alias
    assert lay(f, 4, 8, f, 4, 8, 8, None, f + 64, 1, None) == w4.ERR_INVALID_ARG
    assert lay(f, 4, 4, f, 4, 8, 8, f, f + 64, 1, None) == w4.ERR_INVALID_ARG     # ldx < d_in
    assert lay(f, 4, 8, f, 4, 4, 8, f, f + 64, 1, None) == w4.ERR_INVALID_ARG     # ldw < d_in
    assert lay(None, 4, 8, f, 4, 8, 8, f, f + 64, 1, None) == w4.ERR_INVALID_ARG  # X missing
    assert lay(f, 4, 8, None, 4, 8, 8, f, f + 64, 1, None) == w4.ERR_INVALID_ARG  # W missing
    assert lay(f, -1, 8, f, 4, 8, 8, f, f + 64, 1, None) == w4.ERR_INVALID_ARG
    assert lay(f, 4, 12, f, 4, 12, 12, f, f + 64, 1, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert lay(f + 8, 4, 8, f, 4, 8, 8, f, f + 64, 1, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert lay(None, 0, 8, None, 0, 8, 8, f, f + 64, 0, None) == w4.OK            # nothing to do
    assert w4._calib_finalize(f, f, 64, 0.0, 4, f, f, f, f, f, None) == w4.ERR_INVALID_ARG   # alpha
    assert w4._calib_finalize(f, f, 64, 1.0, 4, f, f, f, f, f, None) == w4.ERR_INVALID_ARG
    assert w4._calib_finalize(f, f, 64, 0.5, 65, f, f, f, f, f, None) == w4.ERR_INVALID_ARG  # k > d_in
    assert w4._calib_finalize(f, f, 64, 0.5, 4, f, f, f, None, f, None) == w4.ERR_INVALID_ARG  # O missing
    assert w4._calib_finalize(f, f, 20000, 0.5, 4, f, f, f, f, f, None) == w4.ERR_UNSUPPORTED_SHAPE


def test_noalloc_limit_and_validation_before_launch():
    # the scratch limit in the header is the one the binding reports
    hdr = open(os.path.join(ROOT, "include", "w4a4.h")).read()
    m = re.search(r"#define W4A4_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == w4.NOALLOC_SCRATCH_BYTES
    assert "no-alloc scratch" in w4.status_string(w4.ERR_SCRATCH_LIMIT)
    # about 12000 tokens of a 5120-wide layer with 32 outliers fit, 12100 do not
    assert w4.workspace_size(12000, 5120, 13824, 32) <= w4.NOALLOC_SCRATCH_BYTES
    assert w4.workspace_size(12100, 5120, 13824, 32) > w4.NOALLOC_SCRATCH_BYTES
    # Pointers here are never dereferenced: each call returns before any CUDA work.
    pw = _raw_pw()
    f = 0x1000
    assert w4._linear_noalloc(f, 8, 63, ctypes.byref(pw), f, 32, None) == w4.ERR_INVALID_ARG
    assert w4._linear_noalloc(f, 8, 64, ctypes.byref(pw), f, 31, None) == w4.ERR_INVALID_ARG
    assert w4._linear_noalloc(None, 8, 64, ctypes.byref(pw), f, 32, None) == w4.ERR_INVALID_ARG
    assert w4._linear_noalloc(f, -1, 64, ctypes.byref(pw), f, 32, None) == w4.ERR_INVALID_ARG
    assert w4._linear_noalloc(f, 0, 64, ctypes.byref(pw), f, 32, None) == w4.OK
    assert w4._linear_noalloc(f, 1 << 20, 64, ctypes.byref(pw), f, 32, None) \
        == w4.ERR_SCRATCH_LIMIT


def test_prep_width_limit():
    # activation prep stages whole rows of at most 16384 bf16 in shared memory
    pw = _raw_pw(d_in=16392, d_out=32, k=4)
    assert w4._prep_act(0x1000, 8, 16392, ctypes.byref(pw), 0x1000, 0x1000, 0x1000, None) \
        == w4.ERR_UNSUPPORTED_SHAPE


def test_packed_image_header_checks():
    # no GPU needed: the header is checked before anything is copied
    import numpy as np
    img = np.zeros(4096, np.uint8)
    d = ctypes.c_int64()
    st = w4._packed_image_info(img.ctypes.data, img.size, ctypes.byref(d), None, None, None)
    assert st == w4.ERR_BAD_IMAGE                       # no magic
    assert w4._packed_image_info(None, 0, None, None, None, None) == w4.ERR_BAD_IMAGE
    img[:8] = np.frombuffer(b"W4A4PKW1", np.uint8)
    assert w4._packed_image_info(img.ctypes.data, img.size, None, None, None, None) \
        == w4.ERR_BAD_IMAGE                             # version 0, zero sizes
    assert "checksum" in w4.status_string(w4.ERR_BAD_IMAGE)
    pw = _raw_pw()
    n = ctypes.c_size_t()
    assert w4._packed_image_size(ctypes.byref(pw), ctypes.byref(n)) == w4.OK
    # header slot + sections, each padded to 64 bytes
    d = w4.get_dims(64, 32, 4)
    sizes = [32 * d.kj_pad // 2, d.sfb_rows * d.nblk, 32 * d.k_pad * 2, 256, 256, 16, 240]
    assert n.value == 256 + sum(-(-x // 64) * 64 for x in sizes)



def test_composite_calls_check_every_step_before_the_first_launch():
    # Pointers here are never dereferenced: the output checks of the GEMM step
    # reject these calls before the prep step (or the upload) is enqueued.
    f = 0x1000
    pw = _raw_pw()                                  # 64 -> 32, k = 4
    ws = w4.workspace_size(8, 64, 32, 4)
    # Y row stride not a multiple of 8 (ldy = 36 >= d_out = 32), Y misaligned
    assert w4._linear(f, 8, 64, ctypes.byref(pw), f, ws, f, 36, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear(f, 8, 64, ctypes.byref(pw), f, ws, f + 8, 32, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear_noalloc(f, 8, 64, ctypes.byref(pw), f, 36, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear_noalloc(f, 8, 64, ctypes.byref(pw), f + 8, 32, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear_noalloc(f + 2, 8, 64, ctypes.byref(pw), f, 32, None) == w4.ERR_UNSUPPORTED_SHAPE
    # the host-buffer layer: misaligned device buffers are caught before the upload
    assert w4._linear_host(f, 8, ctypes.byref(pw), f + 8, f, ws, f, f, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear_host(f, 8, ctypes.byref(pw), f, f, ws, f + 8, f, None) == w4.ERR_UNSUPPORTED_SHAPE
    assert w4._linear_host(f, 8, ctypes.byref(pw), f, f + 8, ws, f, f, None) == w4.ERR_UNSUPPORTED_SHAPE


def test_binding_rejects_what_is_not_bf16_rows():
    import torch
    X = torch.zeros(8, 64, dtype=torch.bfloat16)
    w4._rows_bf16(X, "x", cuda=False)                   # dense host rows pass
    for bad in (X.t(), X.float(), X[:, ::2], X.reshape(-1)):
        with pytest.raises(w4.W4A4Error) as e:
            w4._rows_bf16(bad, "x", cuda=False)
        assert e.value.status == w4.ERR_INVALID_ARG
    with pytest.raises(w4.W4A4Error) as e:
        w4._rows_bf16(X, "x")                           # host memory where device rows are read
    assert e.value.status == w4.ERR_INVALID_ARG


def test_fault_hook_validates_before_touching_the_device():
    # unknown mask bits and limits above the default are refused before any CUDA call
    assert w4._test_fault(2, 0) == w4.ERR_INVALID_ARG
    assert w4._test_fault(1, 3_000_000_000) == w4.ERR_INVALID_ARG
    assert "inf or NaN" in w4.status_string(w4.ERR_NONFINITE_CALIB)


def test_import_fails_loudly_without_the_library(tmp_path):
    """A copy of the package without libw4a4.so refuses to import (no
    fallback path of any kind)."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.dirname(w4.__file__)
    dst = tmp_path / "w4a4_mxfp4_outlier_b200"
    dst.mkdir()
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            shutil.copy(os.path.join(pkg, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import w4a4_mxfp4_outlier_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libw4a4.so is not built" in r.stderr
