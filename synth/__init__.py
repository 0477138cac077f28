"""Seeded synthetic inputs for the W4A4 dual-branch linear.

This module is shared by the CPU oracle tests, the GPU parity tests, the
benchmark and the smoke check.  It produces *inputs only* (activations X and
weights W, as bfloat16 tensors) and the workload table; it contains none of
the method's arithmetic (no smoothing, no outlier selection, no quantisation).

The real calibration data (OpenS2V-5M batches) and the real model weights
(Wan2.2-I2V-A14B FFN layers) are not available, so these generators stand in
for them.  They reproduce the statistics the W4A4 review page reports in its
"Wan2.2 FFN activations are heavy tailed" observation (section 3.1): a few
activation channels whose column maximum exceeds 6.0, a body with a visible
tail beyond |x| > 1.5, and weight columns whose maximum stays below 0.6.

Recipe (all generation is done in float32, then rounded to bfloat16 with
round-to-nearest-even by ``Tensor.to(torch.bfloat16)``):

* Every tensor has its own ``torch.Generator`` seeded from
  ``(seed, tensor_id, chunk)``; rows are generated in fixed chunks of
  ``CHUNK_ROWS`` so the values do not depend on how much memory is free.
* Outlier channels: a seeded random subset of ``n_out`` columns; each gets a
  seeded multiplier drawn uniformly from ``[lo, hi]``.  Other columns get 1.
* ``normal``:  x = sigma * z,                z ~ N(0, 1)
* ``student3``: x = sigma * z / sqrt(c / 3), c = z1^2 + z2^2 + z3^2
  (a Student-t with 3 degrees of freedom)
* ``gelu``:    x = GELU(z) with the exact erf form, z ~ N(0, 1)
* weights:     w = clamp(sigma * z, -0.59375, 0.59375); 0.59375 is the
  largest bfloat16 value below 0.6.

Generation runs on whatever device is asked for; the CUDA and CPU random
streams of torch differ, so a test generates once and hands the *same*
tensor to both the library and the oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

CHUNK_ROWS = 2048
W_CLIP = 0.59375

# tensor ids
_TID_X = 1
_TID_W = 2
_TID_XCOLS = 3


def _gen(seed: int, tid: int, chunk: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 10_007 + chunk) % (2**62))
    return g


@dataclasses.dataclass(frozen=True)
class XSpec:
    """Distribution of one activation matrix [T, d_in]."""
    body: str            # "normal" | "student3" | "gelu"
    sigma: float         # body scale (ignored for gelu)
    n_out: int           # number of outlier channels
    lo: float            # outlier multiplier range
    hi: float


@dataclasses.dataclass(frozen=True)
class WSpec:
    sigma: float


@dataclasses.dataclass(frozen=True)
class Layer:
    """One projection: Y[T, d_out] = X[T, d_in] W[d_out, d_in]^T."""
    name: str
    T: int
    d_in: int
    d_out: int
    alpha: float
    k: int
    layout: int          # 0 = 32x1 K-major scale stripes, 1 = 32x32 tiles, 2 = 128x1 stripes
    x: XSpec
    w: WSpec
    seed: int = 0

    @property
    def flops(self) -> float:
        """Effective FLOPs, 2*T*d_in*d_out (outlier columns counted at the 4-bit rate)."""
        return 2.0 * self.T * self.d_in * self.d_out

    def with_(self, **kw) -> "Layer":
        return dataclasses.replace(self, **kw)


X_TINY = XSpec("normal", 0.3, 8, 10.0, 25.0)
X_UP = XSpec("student3", 0.3, 51, 8.0, 30.0)        # 1% of 5120 channels
X_DOWN = XSpec("gelu", 1.0, 69, 10.0, 20.0)         # 0.5% of 13824 channels
W_UP = WSpec(0.02)
W_DOWN = WSpec(0.015)

TINY = Layer("tiny", 256, 512, 512, 0.5, 8, 0, X_TINY, WSpec(0.02))
FFN0 = Layer("ffn0_T4096", 4096, 5120, 13824, 0.6, 32, 0, X_UP, W_UP)
FFN2 = Layer("ffn2_T4096", 4096, 13824, 5120, 0.7, 64, 0, X_DOWN, W_DOWN)
FULL_UP = Layer("full_up_T57600", 57600, 5120, 13824, 0.6, 32, 0, X_UP, W_UP)
FULL_DOWN = Layer("full_down_T57600", 57600, 13824, 5120, 0.7, 64, 0, X_DOWN, W_DOWN)


def sweep_layers():
    """The sweep at T=16384 on the up-projection shape: k x weight-scale layout
    (32x1, 32x32, 128x1) x alpha."""
    out = []
    for k in (0, 16, 64, 256):
        for layout in (0, 1, 2):
            for alpha in (0.5, 0.7):
                out.append(Layer(f"sweep_k{k}_l{layout}_a{alpha}", 16384, 5120, 13824,
                                 alpha, k, layout, X_UP, W_UP))
    return out


MID_UP = Layer("mid_up_T16384", 16384, 5120, 13824, 0.6, 32, 0, X_UP, W_UP)
MID_DOWN = FULL_DOWN.with_(name="mid_down_T16384", T=16384)

WORKLOADS = {
    "tiny": [TINY],
    "ffn0": [FFN0],
    "ffn2": [FFN2],
    "full": [FULL_UP, FULL_DOWN],
    "full_up": [FULL_UP],
    "full_down": [FULL_DOWN],
    "mid_up": [MID_UP],
    "mid_down": [MID_DOWN],
    "sweep": sweep_layers(),
}


def _outlier_columns(spec: XSpec, d_in: int, seed: int, device):
    g = _gen(seed, _TID_XCOLS, 0, "cpu")
    n = min(spec.n_out, d_in)
    cols = torch.randperm(d_in, generator=g)[:n]
    mult = torch.ones(d_in, dtype=torch.float32)
    mult[cols] = spec.lo + (spec.hi - spec.lo) * torch.rand(n, generator=g)
    return cols.sort().values.to(device), mult.to(device)


def outlier_columns(spec: XSpec, d_in: int, seed: int = 0):
    """The planted outlier channel indices (ascending), for generator checks."""
    return _outlier_columns(spec, d_in, seed, "cpu")[0]


def gen_x(spec: XSpec, T: int, d_in: int, seed: int = 0, device="cpu",
          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Activation matrix [T, d_in], bfloat16, row-major."""
    _, mult = _outlier_columns(spec, d_in, seed, device)
    if out is None:
        out = torch.empty((T, d_in), dtype=torch.bfloat16, device=device)
    for c, r0 in enumerate(range(0, T, CHUNK_ROWS)):
        r1 = min(T, r0 + CHUNK_ROWS)
        g = _gen(seed, _TID_X, c, device)
        z = torch.randn((r1 - r0, d_in), generator=g, device=device, dtype=torch.float32)
        if spec.body == "normal":
            v = spec.sigma * z
        elif spec.body == "student3":
            c3 = torch.zeros_like(z)
            for _ in range(3):
                c3 += torch.randn(z.shape, generator=g, device=device, dtype=torch.float32).square_()
            v = spec.sigma * z / torch.sqrt(c3 / 3.0)
        elif spec.body == "gelu":
            v = torch.nn.functional.gelu(z, approximate="none")
        else:
            raise ValueError(spec.body)
        out[r0:r1] = (v * mult).to(torch.bfloat16)
    return out


def gen_w(spec: WSpec, d_out: int, d_in: int, seed: int = 1, device="cpu") -> torch.Tensor:
    """Weight matrix [d_out, d_in] (row n is output channel n), bfloat16."""
    out = torch.empty((d_out, d_in), dtype=torch.bfloat16, device=device)
    for c, r0 in enumerate(range(0, d_out, CHUNK_ROWS)):
        r1 = min(d_out, r0 + CHUNK_ROWS)
        g = _gen(seed, _TID_W, c, device)
        z = torch.randn((r1 - r0, d_in), generator=g, device=device, dtype=torch.float32)
        out[r0:r1] = (spec.sigma * z).clamp_(-W_CLIP, W_CLIP).to(torch.bfloat16)
    return out


def gen_layer(layer: Layer, device="cpu"):
    """(X, W) for a layer; X uses seed ``layer.seed``, W uses ``layer.seed + 1``."""
    X = gen_x(layer.x, layer.T, layer.d_in, layer.seed, device)
    W = gen_w(layer.w, layer.d_out, layer.d_in, layer.seed + 1, device)
    return X, W


def sample_rows(T: int, n: int, seed: int = 7):
    """A seeded sorted subset of row indices used where the oracle samples rows."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    if n >= T:
        return torch.arange(T)
    return torch.randperm(T, generator=g)[:n].sort().values


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)

