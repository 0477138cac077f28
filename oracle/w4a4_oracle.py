"""CPU oracle for the W4A4 dual-branch linear (test infrastructure only).

This module is the independent, slow, plain-numpy statement of what the GPU
path computes.  It is imported only by ``tests/``, by ``smoke()`` in
``__graft_entry__.py`` and by the CPU-baseline leg of ``bench.py``; the
library and its Python binding never import it, and it shares no code,
table or constant generator with them.

Source of the method: the paper-review page "W4A4 Quantization for Inference
on Wan2.2-I2V-A14B (ICME 2026 Challenge)" (xllm-io paper review), cited below
as [review] with its section and equation:

* [review §3.2, eq. "Y = (X ⊘ s)(s ⊙ W)"]  the SmoothQuant fold;
* [review §3.2, eq. "s_j"]  s_j = act_scale_j^α / weight_scale_j^(1-α);
* [review §3.2, last paragraph]  s is folded into the weights offline, and at
  inference the activations are divided by s before 4-bit quantisation;
* [review §3.3, eq. "score_j"]  score_j = max_t |x_tj|, top-k columns form
  the static outlier set O, J is the complement;
* [review §3.3, eq. "Y = X_J W^(q)_J + X_O W^(hp)_O"]  the dual-branch sum;
* [review §3.4]  block-wise weight scales (32x32 tiles or K-major stripes),
  exponent stored beside the 4-bit payload;
* [review §3.5]  smoothing comes before splitting.

The pages do not bit-specify MXFP4.  The element and scale encodings follow
the OCP Microscaling (MX) v1.0 definitions that the task fixes: E2M1
elements {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit, one E8M0 scale per
32 consecutive K-elements, shared exponent floor(log2 amax) - 2 (2 is the
largest E2M1 exponent), round-half-to-even, saturation at ±6.

Readings taken where the pages are silent (each is also listed in the design
notes):

* act_scale / weight_scale are per-channel absolute maxima;
* scales are clamped below at 1e-5 before the power;
* online smoothing multiplies by inv_s = fl32(1 / s) (one IEEE multiply);
* the score is taken on the smoothed activations (§3.5: smoothing first);
* ties in the top-k go to the lower column index; O and J are ascending;
* J is compacted (O columns dropped) before the 1x32 MX blocks are formed;
  the last block is completed with zeros;
* an all-zero block gets scale code 0 (2^-127) and +-0 codes; the sign of
  zero is kept (code 0x8 for -0);
* the high-precision branch is bfloat16 with round-to-nearest-even;
* nibble order: element 2i in bits [3:0] of byte i, 2i+1 in bits [7:4];
* non-finite values follow IEEE float32 arithmetic and the E8M0 encoding:
  v = fl32(x * inv_s) is +-inf for an infinite x or a product beyond the
  float32 range and NaN for a NaN x; a block's amax is the NaN-propagating
  maximum of |v|; amax = NaN gives scale code 0xFF (E8M0's NaN, the one code
  that marks a whole block as NaN) and all-zero element codes; amax = +inf
  gives e = clamp(floor(log2 inf) - 2) = 127 (code 254), infinities saturate
  to +-6 and finite elements take v * 2^-127 on the E2M1 grid; the bf16
  branch keeps +-inf and writes every NaN as 0x7FC0 (the quiet NaN without
  payload: IEEE does not fix a NaN's sign or payload);
* calibration magnitudes must be finite: s_j is undefined for an infinite or
  NaN magnitude, and the oracle refuses to compute it.

Precision: bf16 inputs are exact in float32.  Every product the method
defines (x * inv_s, w * s) is one float32 multiply with round-to-nearest
even, as the GPU takes it, because it decides integer codes; s itself is
computed in float64 and rounded once; the final product is float64.

Parity pins for every function are in tests/test_oracle_*.py.
"""
from __future__ import annotations

import numpy as np

# E2M1 magnitudes indexed by the 3-bit magnitude code (OCP MX v1.0, FP4 E2M1).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_EMAX = 2          # exponent of the largest normal E2M1 value (6 = 1.5 * 2^2)
MX_BLOCK = 32          # elements sharing one E8M0 scale
SCALE_FLOOR = 1e-5     # lower clamp on calibration magnitudes (our constant)
E8M0_BIAS = 127

LAYOUT_32x1 = 0        # one scale per 32 consecutive K of one output row
LAYOUT_32x32 = 1       # one scale per 32 (rows) x 32 (K) tile
LAYOUT_128x1 = 2       # one scale per 128 consecutive K of one output row (4 MX blocks)


# ----------------------------------------------------------------------------
# bfloat16 helpers (plain definitions)
# ----------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 values (exact widening)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even;
    +-inf stay +-inf, every NaN becomes 0x7FC0 (quiet, no payload)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    return np.where(nan, np.uint16(0x7FC0), r)


# ----------------------------------------------------------------------------
# FFN activation between the two projections
# ----------------------------------------------------------------------------
# The review quantises both FFN projections of the Wan2.2 DiT (ffn.0 and
# ffn.2, §3.1/§3.5); between them the FFN applies GELU (tanh form), which the
# pages do not write out.  The fused up->down step feeds the down projection
# with X_down = bf16_rn(gelu(y)) for the bf16 value y = bf16(Y_up): the bf16
# number nearest the exact value
#
#   gelu(y) = 0.5 y (1 + tanh(u)) = y / (1 + exp(-2u)),  u = sqrt(2/pi) (y + 0.044715 y^3),
#
# ties to even.  That is a function of the 16-bit input with a plain
# definition, so it does not depend on how a kernel evaluates it.  The oracle
# evaluates the second form in float64 (no cancellation for negative y) and
# rounds that once to bf16.  Where the float64 value lies so close to a bf16
# rounding boundary that its own error could decide the rounding (it happens
# for the smallest inputs: gelu(y) = y/2 + O(y^2) with y/2 a bf16 midpoint),
# it recomputes the value with 100 significant digits and decides by exact
# comparison with the boundary (the usual correct-rounding strategy).

_SQRT_2_OVER_PI = np.sqrt(2.0 / np.pi)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns, round to nearest, ties to even, in one
    step (no intermediate float32 rounding).  bf16 keeps 8 significant bits
    down to 2^-126 and a fixed quantum of 2^-133 below (subnormals)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        _, e = np.frexp(a)                                 # a = m 2^e, m in [0.5, 1)
        E = np.maximum(e.astype(np.int64) - 1, -126)       # binade exponent, floored at the subnormals
        q = np.ldexp(1.0, (E - 7).astype(np.int32))        # quantum of that binade
        n = np.rint(a / q)                                 # exact scaling; rint ties to even
        v = n * q
        v = np.where(v > 3.3895313892515355e38, np.inf, v)   # beyond the largest bf16: inf
        v = np.where(np.isfinite(a), v, a)
        v = np.where(a == 0.0, 0.0, v)
    r = np.copysign(v, x).astype(np.float32)               # exact: v is a bf16 value
    bits = (r.view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), bits)


def _bf16_quantum(a: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 values around |a| > 0 (2^-133 below 2^-126)."""
    _, e = np.frexp(a)
    return np.ldexp(1.0, (np.maximum(e.astype(np.int64) - 1, -126) - 7).astype(np.int32))


def _gelu_bf16_exact(yv: float) -> int:
    """bf16 bits of gelu(yv), decided with 100-digit arithmetic."""
    import mpmath
    with mpmath.workdps(100):
        y = mpmath.mpf(yv)
        u = mpmath.sqrt(2 / mpmath.pi) * (y + mpmath.mpf("0.044715") * y ** 3)
        g = y / (1 + mpmath.exp(-2 * u))
        a = abs(g)
        q = mpmath.mpf(float(_bf16_quantum(np.array([float(a)]))[0]))
        n = int(mpmath.floor(a / q))
        mid = (n + mpmath.mpf(0.5)) * q
        if a > mid or (a == mid and n % 2 == 1):
            n += 1
        v = float(n * q)                         # exact: a bf16 value
    return int(f64_to_bf16_bits(np.array([-v if g < 0 or (g == 0 and yv < 0) else v]))[0])


def gelu_bf16(y: np.ndarray) -> np.ndarray:
    """bf16_rn(gelu(y)) for bf16-exact float32 y, as float32 (see above).
    Non-finite inputs follow the float64 formula: +inf -> +inf, -inf and NaN
    -> NaN."""
    yf = np.asarray(y, dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):         # signalling NaNs warn on widening
        yd = yf.astype(np.float64)
        u = _SQRT_2_OVER_PI * (yd + 0.044715 * (yd * yd * yd))
        g = yd / (1.0 + np.exp(-2.0 * u))
    bits = f64_to_bf16_bits(g)
    # float64 carries ~2^-45 of a bf16 quantum of error here; look again at
    # every value within 2^-20 quanta of a rounding boundary
    a = np.abs(g)
    check = np.isfinite(a) & (a > 0) & (a < 3.3e38)
    with np.errstate(divide="ignore", invalid="ignore"):
        frac = np.where(check, a / np.where(check, _bf16_quantum(np.where(check, a, 1.0)), 1.0), 0.0)
    near = check & (np.abs(frac - np.floor(frac) - 0.5) < 2.0 ** -20)
    if near.any():
        flat_bits = bits.reshape(-1)
        flat_y = yd.reshape(-1)
        for i in np.flatnonzero(near.reshape(-1)):
            flat_bits[i] = _gelu_bf16_exact(float(flat_y[i]))
        bits = flat_bits.reshape(bits.shape)
    return bf16_bits_to_f32(bits)


def ffn_hidden(Y_up: np.ndarray) -> np.ndarray:
    """X_down = bf16_rn(gelu(Y_up)) for bf16-exact float32 Y_up."""
    return gelu_bf16(Y_up)


# ----------------------------------------------------------------------------
# Calibration  [review §3.2 "collect per-channel magnitudes"; §3.1]
# ----------------------------------------------------------------------------

def col_absmax(A: np.ndarray, running: np.ndarray | None = None) -> np.ndarray:
    """Per-column max |A[:, j]| as float32, optionally folded into a running max.

    For activations A = X [T, d_in] this is act_scale; for weights stored
    [d_out, d_in] it is weight_scale (the magnitude of input channel j over
    all output channels).  A max of absolute values is exact.
    """
    m = np.max(np.abs(A.astype(np.float32)), axis=0) if A.shape[0] else \
        np.zeros(A.shape[1], np.float32)
    if running is not None:
        m = np.maximum(m, running)
    return m.astype(np.float32)


def smoothing_factors(act_scale: np.ndarray, w_scale: np.ndarray, alpha: float):
    """s_j = act_scale_j^alpha / weight_scale_j^(1-alpha)  [review §3.2, eq. s_j].

    Computed in float64 from the float32 scales (clamped below at 1e-5),
    rounded once to float32.  inv_s = fl32(1 / s) is what the online path
    multiplies by.  Returns (s, inv_s) as float32 arrays.
    """
    if not (np.all(np.isfinite(act_scale)) and np.all(np.isfinite(w_scale))):
        raise ValueError("calibration magnitudes must be finite: s_j is undefined for inf or NaN")
    a = np.maximum(act_scale.astype(np.float64), SCALE_FLOOR)
    w = np.maximum(w_scale.astype(np.float64), SCALE_FLOOR)
    s64 = np.power(a, float(alpha)) / np.power(w, 1.0 - float(alpha))
    s = s64.astype(np.float32)
    inv_s = (1.0 / s.astype(np.float64)).astype(np.float32)
    return s, inv_s


def smooth_activation(X: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    """X ⊘ s, taken as X * inv_s per column j  [review §3.2, eq. fold and last
    paragraph].  Keeps the dtype of its arguments, so float32 inputs give the
    float32 products the quantiser sees and float64 inputs give the exact fold."""
    return X * inv_s[None, :]


def fold_weight(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """s ⊙ W for W stored [d_out, d_in]: input channel j (a column here, a row
    of the pages' d_in x d_out W) is multiplied by s_j  [review §3.2, eq. fold]."""
    return W * s[None, :]


def outlier_scores(X: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    """score_j = max_t |x̃_tj| on the smoothed activations x̃ = fl32(x * inv_s)
    [review §3.3, eq. score_j; §3.5 smoothing before splitting]."""
    V = smooth_activation(X.astype(np.float32), inv_s.astype(np.float32))
    return np.max(np.abs(V), axis=0).astype(np.float32)


def select_outliers(score: np.ndarray, k: int):
    """Static top-k outlier set O and its complement J  [review §3.3].

    Columns are ranked by descending score; equal scores go to the lower
    index.  Returns (O, J) as ascending int32 arrays.
    """
    d = score.shape[0]
    if not 0 <= k <= d:
        raise ValueError("k out of range")
    idx = np.arange(d)
    order = np.lexsort((idx, -score.astype(np.float64)))
    O = np.sort(order[:k]).astype(np.int32)
    J = np.sort(order[k:]).astype(np.int32)
    return O, J


# ----------------------------------------------------------------------------
# MXFP4 encoding (OCP MX v1.0 semantics; the pages name MXFP4 but do not
# bit-specify it)
# ----------------------------------------------------------------------------

def mx_shared_exponent(amax: np.ndarray) -> np.ndarray:
    """e = floor(log2 amax) - 2 clamped to [-127, 127]; e = -127 for amax = 0;
    e = 127 for amax = +inf (floor(log2 inf) is +inf, which the clamp takes to
    127).  A NaN amax has no exponent; the caller codes such a block as NaN.

    floor(log2 amax) is read exactly from frexp (amax = m 2^ex, m in [0.5,1)).
    """
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(np.where(np.isfinite(amax), amax, 1.0))
    e = ex.astype(np.int64) - 1 - E2M1_EMAX
    e = np.where(amax == 0.0, -E8M0_BIAS, e)
    e = np.where(np.isposinf(amax), 127, e)
    return np.clip(e, -127, 127)


def e2m1_codes(q: np.ndarray) -> np.ndarray:
    """Round float32 values to E2M1, nearest with ties to the even code,
    saturating at 6.  Returns 4-bit codes (bit 3 = sign, taken from the sign
    bit of q, so -0 -> 0x8)."""
    # saturate first: anything beyond the largest grid value maps to it
    a = np.minimum(np.abs(np.asarray(q, dtype=np.float64)), E2M1_GRID[-1])
    d = np.abs(a[..., None] - E2M1_GRID)          # exact for float32 inputs
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    even = (np.arange(8) % 2) == 0
    pick = np.where((cand & even).any(-1), (cand & even).argmax(-1), cand.argmax(-1))
    sign = np.signbit(np.asarray(q, dtype=np.float32)).astype(np.int64)
    return (pick | (sign << 3)).astype(np.uint8)


def mxfp4_quantize_blocks(V: np.ndarray, block_amax: np.ndarray | None = None):
    """Quantise float32 values V[..., 32] block-wise.

    Each trailing 32-vector is one MX block.  ``block_amax`` (shape V.shape[:-1])
    overrides the per-block amax, which is how a 32x32 tile shares one scale.
    Returns (scale_codes uint8 [...], codes uint8 [..., 32]).
    """
    V = np.asarray(V, dtype=np.float32)
    if block_amax is None:
        block_amax = np.max(np.abs(V), axis=-1)           # NaN if the block holds a NaN
    nan_block = np.isnan(block_amax)
    e = mx_shared_exponent(np.where(nan_block, 0.0, block_amax))
    # q = v 2^-e is exact in float32 except below 2^-126 (only for e = 127),
    # where it rounds to a subnormal: far below 0.25, the smallest rounding
    # boundary of the E2M1 grid, so the codes are those of the exact q
    with np.errstate(under="ignore", over="ignore", invalid="ignore"):
        q = np.ldexp(V, (-e)[..., None].astype(np.int32)).astype(np.float32)
        codes = e2m1_codes(q)
    codes = np.where(nan_block[..., None], np.uint8(0), codes).astype(np.uint8)
    scale = np.where(nan_block, 0xFF, e + E8M0_BIAS).astype(np.uint8)
    return scale, codes


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """codes[..., 2m] (4-bit) -> bytes[..., m]; element 2i -> bits [3:0]."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    b = b.astype(np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def e2m1_value(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.int64)
    v = E2M1_GRID[c & 7]
    return np.where(c & 8, -v, v)


def dequant_mxfp4(packed: np.ndarray, sf: np.ndarray, ncols: int | None = None) -> np.ndarray:
    """packed [rows, K/2] bytes and sf [rows, K/32] E8M0 -> float64 [rows, K]."""
    codes = unpack_nibbles(packed)
    K = codes.shape[-1]
    scale = np.ldexp(1.0, sf.astype(np.int64) - E8M0_BIAS)          # 2^(sf-127)
    scale = np.where(sf == 0xFF, np.nan, scale)                      # E8M0 0xFF is NaN
    vals = e2m1_value(codes) * np.repeat(scale, MX_BLOCK, axis=-1)[..., :K]
    return vals if ncols is None else vals[..., :ncols]


def _pad_cols(A: np.ndarray, ncols: int) -> np.ndarray:
    if A.shape[1] == ncols:
        return A
    out = np.zeros((A.shape[0], ncols), dtype=A.dtype)
    out[:, :A.shape[1]] = A
    return out


def n_blocks(kj: int) -> int:
    return -(-kj // MX_BLOCK)


# ----------------------------------------------------------------------------
# Online activation preparation  [review §3.2 last paragraph; §3.3 eq. Y]
# ----------------------------------------------------------------------------

def prep_activation(X: np.ndarray, inv_s: np.ndarray, O: np.ndarray, J: np.ndarray,
                    row_chunk: int = 512):
    """Divide by s (multiply by inv_s), split columns into O and J, quantise J.

    X: float32 values [T, d_in] (bf16-exact).  Returns a dict with
      aq   uint8 [T, nblk*16]   packed E2M1 codes of the compacted J columns
      sfa  uint8 [T, nblk]      E8M0 scale codes, row-major (canonical order)
      xo   uint16 [T, k]        bfloat16 bits of the smoothed O columns
    """
    T = X.shape[0]
    kj = J.shape[0]
    nb = n_blocks(kj)
    aq = np.zeros((T, nb * 16), np.uint8)
    sfa = np.zeros((T, nb), np.uint8)
    xo = np.zeros((T, O.shape[0]), np.uint16)
    inv_s = inv_s.astype(np.float32)
    for r0 in range(0, T, row_chunk):
        r1 = min(T, r0 + row_chunk)
        with np.errstate(over="ignore", invalid="ignore"):
            V = smooth_activation(X[r0:r1].astype(np.float32), inv_s)   # fl32 products (may be +-inf)
        xo[r0:r1] = f32_to_bf16_bits(V[:, O])
        if nb:
            VJ = _pad_cols(V[:, J], nb * MX_BLOCK).reshape(r1 - r0, nb, MX_BLOCK)
            sc, codes = mxfp4_quantize_blocks(VJ)
            sfa[r0:r1] = sc
            aq[r0:r1] = pack_nibbles(codes.reshape(r1 - r0, nb * MX_BLOCK))
    return {"aq": aq, "sfa": sfa, "xo": xo}


# ----------------------------------------------------------------------------
# Offline weight packing  [review §3.2 fold; §3.3 split; §3.4 block packing]
# ----------------------------------------------------------------------------

def pack_weight(W: np.ndarray, s: np.ndarray, O: np.ndarray, J: np.ndarray,
                layout: int = LAYOUT_32x1, row_chunk: int = 512):
    """Fold s into W, split off the O rows (columns here) in bf16, MXFP4-pack J.

    W: float32 values [d_out, d_in] (bf16-exact).  Returns a dict with
      wq    uint8 [d_out, nblk*16]  packed codes of the compacted J columns
      sfb   uint8 [d_out, nblk]     E8M0 codes (32x32: the tile's code repeated
                                    on each of its 32 rows; 128x1: the stripe's
                                    code repeated on its 4 blocks)
      w_hp  uint16 [d_out, k]       bfloat16 bits of the folded O columns
    Rows are processed in chunks (a multiple of 32) only to bound memory.
    """
    if layout not in (LAYOUT_32x1, LAYOUT_32x32, LAYOUT_128x1):
        raise ValueError("unknown layout")
    d_out = W.shape[0]
    kj = J.shape[0]
    nb = n_blocks(kj)
    s = s.astype(np.float32)
    wq = np.zeros((d_out, nb * 16), np.uint8)
    sfb = np.zeros((d_out, nb), np.uint8)
    w_hp = np.zeros((d_out, O.shape[0]), np.uint16)
    for r0 in range(0, d_out, row_chunk):
        r1 = min(d_out, r0 + row_chunk)
        with np.errstate(over="ignore", invalid="ignore"):
            Wf = fold_weight(W[r0:r1].astype(np.float32), s).astype(np.float32)   # fl32 products
        w_hp[r0:r1] = f32_to_bf16_bits(Wf[:, O])
        if not nb:
            continue
        WJ = _pad_cols(Wf[:, J], nb * MX_BLOCK).reshape(r1 - r0, nb, MX_BLOCK)
        if layout == LAYOUT_32x1:
            sc, codes = mxfp4_quantize_blocks(WJ)
        elif layout == LAYOUT_128x1:
            # [review §3.4] "128x1 K-major stripe": one amax per 128 consecutive
            # compacted K of a row, i.e. per 4 consecutive MX blocks from p = 0;
            # a last partial stripe is completed with zero blocks
            amax_blocks = np.max(np.abs(WJ), axis=-1)                        # [rows, nb]
            padb = (-nb) % 4
            amax_blocks = np.concatenate(
                [amax_blocks, np.zeros((r1 - r0, padb), np.float32)], axis=1)
            stripe = amax_blocks.reshape(r1 - r0, -1, 4).max(axis=-1)        # [rows, stripes]
            sc, codes = mxfp4_quantize_blocks(WJ, np.repeat(stripe, 4, axis=1)[:, :nb])
        else:
            # one amax per 32 rows x 32 columns; rows past d_out count as zeros
            amax_rows = np.max(np.abs(WJ), axis=-1)                          # [rows, nb]
            pad = (-(r1 - r0)) % 32
            amax_rows = np.concatenate([amax_rows, np.zeros((pad, nb), np.float32)], axis=0)
            tile_amax = amax_rows.reshape(-1, 32, nb).max(axis=1)            # [tiles, nb]
            per_row = np.repeat(tile_amax, 32, axis=0)[:r1 - r0]
            sc, codes = mxfp4_quantize_blocks(WJ, per_row)
        sfb[r0:r1] = sc
        wq[r0:r1] = pack_nibbles(codes.reshape(r1 - r0, nb * MX_BLOCK))
    return {"wq": wq, "sfb": sfb, "w_hp": w_hp}


# ----------------------------------------------------------------------------
# Dual-branch product  [review §3.3, eq. Y = X_J W^(q)_J + X_O W^(hp)_O]
# ----------------------------------------------------------------------------

def dual_branch_product(aq, sfa, xo, wq, sfb, w_hp) -> np.ndarray:
    """Y[t, n] = sum_p deq(Aq)[t,p] deq(Wq)[n,p] + sum_i X_O[t,i] W_hp[n,i], float64."""
    A = dequant_mxfp4(aq, sfa)
    B = dequant_mxfp4(wq, sfb)
    Y = A @ B.T
    if xo.shape[1]:
        Y = Y + bf16_bits_to_f32(xo).astype(np.float64) @ bf16_bits_to_f32(w_hp).astype(np.float64).T
    return Y


# ----------------------------------------------------------------------------
# Whole path
# ----------------------------------------------------------------------------

def calibrate(X_batches, W: np.ndarray, alpha: float, k: int):
    """Calibration and outlier selection over one or more activation batches."""
    if isinstance(X_batches, np.ndarray):
        X_batches = [X_batches]
    act = None
    for Xb in X_batches:
        act = col_absmax(Xb, act)
    wsc = col_absmax(W)
    s, inv_s = smoothing_factors(act, wsc, alpha)
    score = None
    for Xb in X_batches:
        sc = outlier_scores(Xb, inv_s)
        score = sc if score is None else np.maximum(score, sc)
    O, J = select_outliers(score, k)
    return {"act_scale": act, "w_scale": wsc, "s": s, "inv_s": inv_s,
            "score": score, "O": O, "J": J}


def linear_reference(X: np.ndarray, W: np.ndarray, alpha: float, k: int,
                     layout: int = LAYOUT_32x1, rows=None, calib=None):
    """The W4A4 dual-branch linear on the CPU.  X [T, d_in], W [d_out, d_in]
    as float32 values.  ``rows`` restricts the product to those rows (the
    calibration still sees all of X).  Returns (Y float64, pieces dict)."""
    c = calib if calib is not None else calibrate(X, W, alpha, k)
    pw = pack_weight(W, c["s"], c["O"], c["J"], layout)
    Xr = X if rows is None else X[rows]
    pa = prep_activation(Xr, c["inv_s"], c["O"], c["J"])
    Y = dual_branch_product(pa["aq"], pa["sfa"], pa["xo"], pw["wq"], pw["sfb"], pw["w_hp"])
    return Y, {**c, **pw, **pa}


def search_layer(X: np.ndarray, W: np.ndarray, alphas, ks, layouts=(LAYOUT_32x1,), X_eval=None):
    """Layer-wise (alpha, k, layout) choice [review sec. 4 table "Layer-wise
    alpha and k"; sec. 6 "next step"; no procedure given]: for every
    candidate the quantised layer's Y on X_eval (default X, calibration on X)
    is compared with the exact float64 product X_eval W^T; the smallest
    relative Frobenius error wins, the smaller k on ties, then the candidate
    listed first (layouts, then k, then alpha, in the order given).
    Returns (best, {candidate: error})."""
    Xe = X if X_eval is None else X_eval
    exact = Xe.astype(np.float64) @ W.astype(np.float64).T
    den = float(np.sum(exact * exact))
    errors = {}
    for layout in layouts:
        for k in ks:
            for alpha in alphas:
                c = calibrate(X, W, alpha, k)
                pw = pack_weight(W, c["s"], c["O"], c["J"], layout)
                pa = prep_activation(Xe, c["inv_s"], c["O"], c["J"])
                Y = dual_branch_product(pa["aq"], pa["sfa"], pa["xo"], pw["wq"], pw["sfb"],
                                        pw["w_hp"])
                errors[(alpha, k, layout)] = float(np.sqrt(np.sum((Y - exact) ** 2) / den)) \
                    if den > 0 else 0.0
    best = min(errors, key=lambda cnd: (errors[cnd], cnd[1]))
    return best, errors


def mma_sf_offset(r, kb, nblk: int):
    """Byte offset of scale (row r, block kb) in the block-scaled MMA layout.

    The layout is the public one for Blackwell block-scaled MMAs (CUTLASS
    ``Sm1xxBlockScaledConfig``): 128-row x 4-block atoms of 512 bytes, atoms
    K-major, inside an atom row r sits at (r % 32) * 16 + ((r % 128) // 32) * 4
    and block kb at kb % 4.  ``nblk`` is the number of blocks per row of the
    buffer (padded to a multiple of 4).  Accepts integers or numpy integer
    arrays.  Used by tests to read GPU scale buffers back into the canonical
    [rows, nblk] order; it is a storage order, not part of the arithmetic.
    """
    atoms_k = -(-nblk // 4)
    return (((r // 128) * atoms_k + kb // 4) * 512 + (r % 32) * 16
            + ((r % 128) // 32) * 4 + kb % 4)
