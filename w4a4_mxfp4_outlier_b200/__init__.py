"""Python binding of libw4a4 (W4A4 dual-branch linear for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libw4a4.so``; torch supplies device memory and streams.  The
functions carry the names of the C entry points in ``include/w4a4.h``
without the ``w4a4_`` prefix.  Importing this module fails loudly when the
shared library is missing (build it with ``python
w4a4_mxfp4_outlier_b200/build.py``); there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libw4a4.so is not built ({LIB_PATH}); run "
                      "`python w4a4_mxfp4_outlier_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_LIMIT,
 ERR_BAD_IMAGE, ERR_NONFINITE_CALIB) = range(8)
NOALLOC_SCRATCH_BYTES = 32 << 20     # W4A4_NOALLOC_SCRATCH_BYTES
SF_32x1_KMAJOR, SF_32x32_TILE, SF_128x1_KMAJOR = 0, 1, 2

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class Dims(ctypes.Structure):
    _fields_ = [(n, _i64) for n in ("d_in", "d_out", "k", "kj", "kj_pad", "nblk", "k_pad", "sfb_rows")]


class WeightBytes(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_size_t), ("sfb", ctypes.c_size_t), ("w_hp", ctypes.c_size_t)]


class PackedWeightC(ctypes.Structure):
    _fields_ = [("d_in", _i64), ("d_out", _i64), ("k", _i64), ("layout", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("wq", _vp), ("sfb", _vp), ("w_hp", _vp),
                ("inv_s", _vp), ("O", _vp), ("jmap", _vp)]


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_st = ctypes.c_int
_abi_version = _sig("w4a4_abi_version", ctypes.c_int)
_status_string = _sig("w4a4_status_string", ctypes.c_char_p, _st)
_num_sms = _sig("w4a4_num_sms", ctypes.c_int)
_get_dims = _sig("w4a4_get_dims", _st, _i64, _i64, _i64, ctypes.POINTER(Dims))
_calib_observe = _sig("w4a4_calib_observe", _st, _vp, _i64, _i64, _i64, _vp, ctypes.c_int, _vp)
_calib_observe_layer = _sig("w4a4_calib_observe_layer", _st, _vp, _i64, _i64, _vp, _i64, _i64, _i64,
                            _vp, _vp, ctypes.c_int, _vp)
_calib_finalize = _sig("w4a4_calib_finalize", _st, _vp, _vp, _i64, ctypes.c_double, _i64,
                       _vp, _vp, _vp, _vp, _vp, _vp)
_weight_sizes = _sig("w4a4_weight_sizes", _st, _i64, _i64, _i64, ctypes.POINTER(WeightBytes))
_pack_weight = _sig("w4a4_pack_weight", _st, _vp, _i64, _vp, ctypes.POINTER(PackedWeightC), _vp)
_workspace_size = _sig("w4a4_workspace_size", _st, _i64, _i64, _i64, _i64,
                       ctypes.POINTER(ctypes.c_size_t))
_prep_act = _sig("w4a4_prep_act", _st, _vp, _i64, _i64, ctypes.POINTER(PackedWeightC), _vp, _vp,
                 _vp, _vp)
_gemm_dual = _sig("w4a4_gemm_dual", _st, _vp, _vp, _vp, _i64, ctypes.POINTER(PackedWeightC), _vp,
                  _i64, _vp)
_linear = _sig("w4a4_linear", _st, _vp, _i64, _i64, ctypes.POINTER(PackedWeightC), _vp,
               ctypes.c_size_t, _vp, _i64, _vp)
_linear_host = _sig("w4a4_linear_host", _st, _vp, _i64, ctypes.POINTER(PackedWeightC), _vp, _vp,
                    ctypes.c_size_t, _vp, _vp, _vp)
_linear_noalloc = _sig("w4a4_linear_noalloc", _st, _vp, _i64, _i64, ctypes.POINTER(PackedWeightC),
                       _vp, _i64, _vp)
_packed_image_size = _sig("w4a4_packed_image_size", _st, ctypes.POINTER(PackedWeightC),
                          ctypes.POINTER(ctypes.c_size_t))
_packed_save = _sig("w4a4_packed_save", _st, ctypes.POINTER(PackedWeightC), _vp, _vp,
                    ctypes.c_size_t, _vp)
_packed_image_info = _sig("w4a4_packed_image_info", _st, _vp, ctypes.c_size_t,
                          ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_i64),
                          ctypes.POINTER(ctypes.c_int32))
_packed_load = _sig("w4a4_packed_load", _st, _vp, ctypes.c_size_t, ctypes.POINTER(PackedWeightC),
                    _vp, _vp)
_gelu_bf16 = _sig("w4a4_gelu_bf16", _st, _vp, _i64, _i64, _i64, _vp, _i64, _vp)
_ffn_link = _sig("w4a4_ffn_link", _st, ctypes.POINTER(PackedWeightC), _vp, _vp, _vp)
_pack_weight_rows = _sig("w4a4_pack_weight_rows", _st, _vp, _i64, _vp, _vp,
                         ctypes.POINTER(PackedWeightC), _vp)
_permute_packed_rows = _sig("w4a4_permute_packed_rows", _st, ctypes.POINTER(PackedWeightC), _vp,
                            ctypes.POINTER(PackedWeightC), _vp)
_gemm_dual_act = _sig("w4a4_gemm_dual_act", _st, _vp, _vp, _vp, _i64, ctypes.POINTER(PackedWeightC),
                      ctypes.POINTER(PackedWeightC), _vp, _vp, _vp, _vp, _vp)
_error_sums = _sig("w4a4_error_sums", _st, _vp, _i64, _vp, _i64, _i64, _i64, _vp, _vp)
_last_error = _sig("w4a4_last_error", _st, _vp, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32))
_test_fault = _sig("w4a4_test_fault", _st, ctypes.c_uint32, ctypes.c_uint64)
FAULT_PREP_SKIP_LOADS = 1           # W4A4_FAULT_PREP_SKIP_LOADS

EXPORTED = [
    "w4a4_abi_version", "w4a4_status_string", "w4a4_num_sms", "w4a4_get_dims",
    "w4a4_calib_observe", "w4a4_calib_observe_layer", "w4a4_calib_finalize", "w4a4_weight_sizes",
    "w4a4_pack_weight",
    "w4a4_workspace_size", "w4a4_prep_act", "w4a4_gemm_dual", "w4a4_linear",
    "w4a4_linear_host", "w4a4_linear_noalloc", "w4a4_last_error",
    "w4a4_packed_image_size", "w4a4_packed_save", "w4a4_packed_image_info", "w4a4_packed_load",
    "w4a4_error_sums", "w4a4_gelu_bf16", "w4a4_ffn_link", "w4a4_pack_weight_rows", "w4a4_permute_packed_rows",
    "w4a4_gemm_dual_act", "w4a4_test_fault",
]


class W4A4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def _check(status: int, what: str):
    if status != OK:
        raise W4A4Error(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _rows_bf16(t: torch.Tensor, what: str, device=None, cuda: bool = True):
    """The library reads a bf16 matrix as rows of contiguous elements with a
    row stride: reject anything else (another dtype, a transposed or
    column-strided view, a tensor on another device) before the call, since
    the C ABI sees only a pointer and a row stride."""
    ok = (t.dtype == torch.bfloat16 and t.dim() == 2 and (t.stride(1) == 1 or t.shape[1] <= 1)
          and t.is_cuda == cuda and (device is None or not cuda or t.device == torch.device(device)))
    if not ok:
        raise W4A4Error(ERR_INVALID_ARG,
                        f"{what}: needs a 2-D bfloat16 {'CUDA' if cuda else 'host'} tensor with "
                        f"unit column stride{' on ' + str(device) if device is not None and cuda else ''}"
                        f" (got {t.dtype}, shape {tuple(t.shape)}, strides {tuple(t.stride())}, "
                        f"{t.device})")
    if not cuda and not t.is_contiguous():
        raise W4A4Error(ERR_INVALID_ARG, f"{what}: host rows must be dense")


def _stream(stream) -> Optional[int]:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def abi_version() -> int:
    return _abi_version()


def status_string(status: int) -> str:
    return _status_string(status).decode()


def num_sms() -> int:
    return _num_sms()


def get_dims(d_in: int, d_out: int, k: int) -> Dims:
    d = Dims()
    _check(_get_dims(d_in, d_out, k, ctypes.byref(d)), "get_dims")
    return d


def weight_sizes(d_in: int, d_out: int, k: int) -> WeightBytes:
    b = WeightBytes()
    _check(_weight_sizes(d_in, d_out, k, ctypes.byref(b)), "weight_sizes")
    return b


def workspace_size(T: int, d_in: int, d_out: int, k: int) -> int:
    n = ctypes.c_size_t()
    _check(_workspace_size(T, d_in, d_out, k, ctypes.byref(n)), "workspace_size")
    return n.value


def calib_observe(A: torch.Tensor, absmax: torch.Tensor, reset: bool, stream=None):
    _rows_bf16(A, "calib_observe", absmax.device)
    rows, cols = A.shape
    _check(_calib_observe(_ptr(A), rows, cols, A.stride(0), _ptr(absmax), int(reset),
                          _stream(stream)), "calib_observe")


def calib_observe_layer(X: torch.Tensor, W: torch.Tensor, act_scale: torch.Tensor,
                        w_scale: torch.Tensor, reset: bool, stream=None):
    """Column absmax of X into act_scale and of W into w_scale, one launch."""
    _rows_bf16(X, "calib_observe_layer", act_scale.device)
    _rows_bf16(W, "calib_observe_layer", act_scale.device)
    if X.shape[1] != W.shape[1]:
        raise W4A4Error(ERR_INVALID_ARG, f"calib_observe_layer: X has {X.shape[1]} columns, "
                        f"W {W.shape[1]}")
    _check(_calib_observe_layer(_ptr(X), X.shape[0], X.stride(0), _ptr(W), W.shape[0], W.stride(0),
                                X.shape[1], _ptr(act_scale), _ptr(w_scale), int(reset),
                                _stream(stream)), "calib_observe_layer")


def calib_finalize(act_scale, w_scale, alpha: float, k: int, s, inv_s, score, O, jmap, stream=None):
    _check(_calib_finalize(_ptr(act_scale), _ptr(w_scale), act_scale.numel(), float(alpha), k,
                           _ptr(s), _ptr(inv_s), _ptr(score), _ptr(O), _ptr(jmap),
                           _stream(stream)), "calib_finalize")


@dataclass
class PackedWeight:
    """Device buffers of one packed layer plus the C record pointing at them."""
    d_in: int
    d_out: int
    k: int
    layout: int
    wq: torch.Tensor
    sfb: torch.Tensor
    w_hp: torch.Tensor
    s: torch.Tensor
    inv_s: torch.Tensor
    score: torch.Tensor
    O: torch.Tensor
    jmap: torch.Tensor
    act_scale: torch.Tensor
    w_scale: torch.Tensor

    @property
    def c(self) -> PackedWeightC:
        return PackedWeightC(self.d_in, self.d_out, self.k, self.layout, 0,
                             _ptr(self.wq) if self.wq.numel() else None,
                             _ptr(self.sfb) if self.sfb.numel() else None,
                             _ptr(self.w_hp) if self.w_hp.numel() else None,
                             _ptr(self.inv_s),
                             _ptr(self.O) if self.O.numel() else None,
                             _ptr(self.jmap) if self.jmap.numel() else None)

    @property
    def dims(self) -> Dims:
        return get_dims(self.d_in, self.d_out, self.k)


def alloc_packed(d_in: int, d_out: int, k: int, layout: int = SF_32x1_KMAJOR, device="cuda") -> PackedWeight:
    b = weight_sizes(d_in, d_out, k)
    u8 = dict(dtype=torch.uint8, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    i32 = dict(dtype=torch.int32, device=device)
    return PackedWeight(d_in, d_out, k, layout,
                        torch.empty(b.wq, **u8), torch.empty(b.sfb, **u8),
                        torch.empty(b.w_hp // 2, dtype=torch.bfloat16, device=device),
                        torch.empty(d_in, **f32), torch.empty(d_in, **f32), torch.empty(d_in, **f32),
                        torch.empty(k, **i32), torch.empty(d_in - k, **i32),
                        torch.empty(d_in, **f32), torch.empty(d_in, **f32))


def pack_weight(W: torch.Tensor, pw: PackedWeight, stream=None):
    _rows_bf16(W, "pack_weight", pw.wq.device)
    c = pw.c
    _check(_pack_weight(_ptr(W), W.stride(0), _ptr(pw.s), ctypes.byref(c), _stream(stream)),
           "pack_weight")


def calibrate(X_batches, W: torch.Tensor, alpha: float, k: int,
              layout: int = SF_32x1_KMAJOR, stream=None) -> PackedWeight:
    """Column absmax of the first activation batch and W (one launch), of the
    further batches (running maximum), calib_finalize, then pack_weight: the
    offline half of the method, all on the device."""
    if isinstance(X_batches, torch.Tensor):
        X_batches = [X_batches]
    d_out, d_in = W.shape
    pw = alloc_packed(d_in, d_out, k, layout, W.device)
    calib_observe_layer(X_batches[0], W, pw.act_scale, pw.w_scale, reset=True, stream=stream)
    for Xb in X_batches[1:]:
        calib_observe(Xb, pw.act_scale, reset=False, stream=stream)
    calib_finalize(pw.act_scale, pw.w_scale, alpha, k, pw.s, pw.inv_s, pw.score,
                   pw.O if k else None, pw.jmap if k < d_in else None, stream=stream)
    pack_weight(W, pw, stream=stream)
    return pw


@dataclass
class ActBuffers:
    aq: torch.Tensor     # uint8 [T, kj_pad/2]
    sfa: torch.Tensor    # uint8, MMA layout
    xo: torch.Tensor     # bf16 [T, k_pad]


def alloc_act(T: int, pw: PackedWeight) -> ActBuffers:
    d = pw.dims
    dev = pw.wq.device
    return ActBuffers(torch.empty((T, d.kj_pad // 2), dtype=torch.uint8, device=dev),
                      torch.empty(((T + 127) // 128 * 128) * d.nblk, dtype=torch.uint8, device=dev),
                      torch.empty((T, d.k_pad), dtype=torch.bfloat16, device=dev))


def _nz(t: torch.Tensor):
    return _ptr(t) if t.numel() else None


def prep_act(X: torch.Tensor, pw: PackedWeight, out: ActBuffers, stream=None):
    _rows_bf16(X, "prep_act", pw.wq.device)
    c = pw.c
    _check(_prep_act(_ptr(X), X.shape[0], X.stride(0), ctypes.byref(c), _nz(out.aq), _nz(out.sfa),
                     _nz(out.xo), _stream(stream)), "prep_act")


def gemm_dual(act: ActBuffers, T: int, pw: PackedWeight, Y: torch.Tensor, stream=None):
    _rows_bf16(Y, "gemm_dual", pw.wq.device)
    c = pw.c
    _check(_gemm_dual(_nz(act.aq), _nz(act.sfa), _nz(act.xo), T, ctypes.byref(c), _ptr(Y),
                      Y.stride(0), _stream(stream)), "gemm_dual")


def linear(X: torch.Tensor, pw: PackedWeight, workspace: torch.Tensor, Y: torch.Tensor, stream=None):
    _rows_bf16(X, "linear", pw.wq.device)
    _rows_bf16(Y, "linear", pw.wq.device)
    c = pw.c
    _check(_linear(_ptr(X), X.shape[0], X.stride(0), ctypes.byref(c), _ptr(workspace),
                   workspace.numel() * workspace.element_size(), _ptr(Y), Y.stride(0),
                   _stream(stream)), "linear")


def linear_host(X_host: torch.Tensor, pw: PackedWeight, X_dev: torch.Tensor, workspace: torch.Tensor,
                Y_dev: torch.Tensor, Y_host: torch.Tensor, stream=None):
    _rows_bf16(X_host, "linear_host", cuda=False)
    _rows_bf16(Y_host, "linear_host", cuda=False)
    for t in (X_dev, Y_dev):
        _rows_bf16(t, "linear_host", pw.wq.device)
        if not t.is_contiguous():
            raise W4A4Error(ERR_INVALID_ARG, "linear_host: device rows must be dense")
    c = pw.c
    _check(_linear_host(_ptr(X_host), X_host.shape[0], ctypes.byref(c), _ptr(X_dev),
                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                        _ptr(Y_dev), _ptr(Y_host), _stream(stream)), "linear_host")


def linear_noalloc(X: torch.Tensor, pw: PackedWeight, Y: torch.Tensor, stream=None):
    """The online layer with the library's fixed scratch array instead of a
    workspace: allocates nothing, for callers that cannot hand over device
    memory.  Problems larger than NOALLOC_SCRATCH_BYTES of workspace raise
    W4A4Error(ERR_SCRATCH_LIMIT); calls overlapping on the GPU must be
    serialised by the caller (they share the array)."""
    _rows_bf16(X, "linear_noalloc", pw.wq.device)
    _rows_bf16(Y, "linear_noalloc", pw.wq.device)
    c = pw.c
    _check(_linear_noalloc(_ptr(X), X.shape[0], X.stride(0), ctypes.byref(c), _ptr(Y), Y.stride(0),
                           _stream(stream)), "linear_noalloc")


def packed_to_bytes(pw: PackedWeight, stream=None) -> bytes:
    """The checkpoint image of a packed layer (see w4a4_packed_save)."""
    c = pw.c
    n = ctypes.c_size_t()
    _check(_packed_image_size(ctypes.byref(c), ctypes.byref(n)), "packed_image_size")
    buf = torch.empty(n.value, dtype=torch.uint8, pin_memory=torch.cuda.is_available())
    _check(_packed_save(ctypes.byref(c), _ptr(pw.s), buf.data_ptr(), n.value, _stream(stream)),
           "packed_save")
    return buf.numpy().tobytes()


def packed_from_bytes(image: bytes, device="cuda", stream=None) -> PackedWeight:
    """Allocates a packed layer on `device` and loads a checkpoint image into
    it.  act_scale, w_scale and score are not part of the image (zeros)."""
    buf = torch.frombuffer(bytearray(image), dtype=torch.uint8)
    d_in, d_out, k, layout = _i64(), _i64(), _i64(), ctypes.c_int32()
    _check(_packed_image_info(buf.data_ptr(), buf.numel(), ctypes.byref(d_in), ctypes.byref(d_out),
                              ctypes.byref(k), ctypes.byref(layout)), "packed_image_info")
    pw = alloc_packed(d_in.value, d_out.value, k.value, layout.value, device)
    for t in (pw.act_scale, pw.w_scale, pw.score):
        t.zero_()
    c = pw.c
    _check(_packed_load(buf.data_ptr(), buf.numel(), ctypes.byref(c), _ptr(pw.s), _stream(stream)),
           "packed_load")
    return pw


def save_packed(pw: PackedWeight, path: str, stream=None):
    with open(path, "wb") as f:
        f.write(packed_to_bytes(pw, stream))


def load_packed(path: str, device="cuda", stream=None) -> PackedWeight:
    with open(path, "rb") as f:
        return packed_from_bytes(f.read(), device, stream)


def test_fault(mask: int, wait_limit_ns: int = 0):
    """Failure-detection test hook (w4a4_test_fault): shorten the device wait
    limit and make the prep producer skip its copies; test_fault(0, 0)
    restores normal operation."""
    _check(_test_fault(mask, wait_limit_ns), "test_fault")


def last_error(clear: bool = True, stream=None):
    bits = ctypes.c_uint32()
    st = _last_error(_stream(stream), int(clear), ctypes.byref(bits))
    return st, bits.value
