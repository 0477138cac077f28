"""Interval bounds for the FFN chain from X (test infrastructure): the set
of down-layer outputs that any up-layer output within a tolerance band can
produce, carried through the bf16 GELU, the smoothing multiply, the MXFP4
quantiser and the down product.  Built from the oracle's own definitions
(each step is monotone, or its extremes are known), so a GPU result can be
checked against an oracle chain that starts from X without using any GPU
value."""
import numpy as np

from oracle import w4a4_oracle as orc


def bf16_round_out(lo, hi):
    """The bf16 grid interval [lo', hi'] with lo' <= lo, hi' >= hi (outward)."""
    lo32 = np.asarray(lo, np.float32)
    hi32 = np.asarray(hi, np.float32)
    def down(x):      # largest bf16 <= x
        b = orc.f32_to_bf16_bits(x)
        v = orc.bf16_bits_to_f32(b)
        step = np.where(v > x, 1, 0).astype(np.int32)
        # one bf16 ulp toward -inf where rounding went up
        bits = b.astype(np.int32)
        bits = np.where(step == 1, np.where(bits & 0x8000, bits + 1, np.where(bits == 0, 0x8001, bits - 1)), bits)
        return orc.bf16_bits_to_f32(bits.astype(np.uint16))
    return down(lo32), -down(-hi32)


def gelu_interval(ylo, yhi):
    """[min, max] of bf16(gelu(y)) over the bf16 values y in [ylo, yhi]: the
    function decreases below y* = -0.7518 and increases above, so the extremes
    sit at the ends or at the bf16 values next to y*."""
    g_lo, g_hi = orc.gelu_bf16(ylo), orc.gelu_bf16(yhi)
    gmin, gmax = np.minimum(g_lo, g_hi), np.maximum(g_lo, g_hi)
    inside = (ylo <= -0.75) & (yhi >= -0.76)
    if inside.any():
        cand = orc.bf16_bits_to_f32(np.arange(0xBF3F, 0xBF43, dtype=np.uint16))   # -0.746 .. -0.762
        gc = orc.gelu_bf16(cand).astype(np.float64)
        for c, g in zip(cand, gc):
            m = inside & (ylo <= c) & (yhi >= c)
            gmin = np.where(m, np.minimum(gmin, g), gmin)
    return gmin, gmax


def mx_interval(vlo, vhi):
    """Bounds of the dequantised MXFP4 values of blocks whose float32 inputs
    lie anywhere in [vlo, vhi] (elementwise, last axis = 32 per block): every
    exponent the block maximum allows, each element rounded at its ends
    (rounding to the E2M1 grid at a fixed exponent is monotone)."""
    amin = np.where((vlo <= 0) & (vhi >= 0), 0.0, np.minimum(np.abs(vlo), np.abs(vhi)))
    amax = np.maximum(np.abs(vlo), np.abs(vhi))
    e_lo = orc.mx_shared_exponent(amin.max(axis=-1))
    e_hi = orc.mx_shared_exponent(amax.max(axis=-1))
    out_lo = np.full(vlo.shape, np.inf)
    out_hi = np.full(vlo.shape, -np.inf)
    for de in range(int((e_hi - e_lo).max()) + 1):
        e = np.minimum(e_lo + de, e_hi)[..., None].astype(np.int32)
        for v in (vlo, vhi):
            q = orc.e2m1_value(orc.e2m1_codes(np.ldexp(v.astype(np.float32), -e).astype(np.float32)))
            d = np.ldexp(q, e)
            out_lo = np.minimum(out_lo, d)
            out_hi = np.maximum(out_hi, d)
    return out_lo, out_hi



def down_interval(Yu, tol, cd, Wd, layout):
    """[Ylo, Yhi] elementwise for the down layer fed bf16(gelu(y)) with y any
    bf16 value within Yu +- tol; cd: the down layer's s, inv_s, O, J."""
    T = Yu.shape[0]
    ylo, yhi = bf16_round_out(Yu - tol, Yu + tol)
    hlo, hhi = gelu_interval(ylo, yhi)
    inv = cd["inv_s"].astype(np.float32)
    vlo = (hlo.astype(np.float32) * inv[None, :]).astype(np.float32)   # fl32, monotone (inv_s > 0)
    vhi = (hhi.astype(np.float32) * inv[None, :]).astype(np.float32)
    J, O = cd["J"], cd["O"]
    nb = orc.n_blocks(J.size)
    pad = lambda a: orc._pad_cols(a, nb * 32).reshape(T, nb, 32)
    alo, ahi = mx_interval(pad(vlo[:, J]), pad(vhi[:, J]))
    alo, ahi = alo.reshape(T, -1), ahi.reshape(T, -1)
    wd = orc.pack_weight(Wd, cd["s"], O, J, layout)
    B = orc.dequant_mxfp4(wd["wq"], wd["sfb"])
    pos, neg = np.maximum(B, 0), np.minimum(B, 0)
    Ylo = alo @ pos.T + ahi @ neg.T
    Yhi = ahi @ pos.T + alo @ neg.T
    if O.size:
        xlo = orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(vlo[:, O])).astype(np.float64)
        xhi = orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(vhi[:, O])).astype(np.float64)
        Bh = orc.bf16_bits_to_f32(wd["w_hp"]).astype(np.float64)
        Ylo += xlo @ np.maximum(Bh, 0).T + xhi @ np.minimum(Bh, 0).T
        Yhi += xhi @ np.maximum(Bh, 0).T + xlo @ np.minimum(Bh, 0).T
    return Ylo, Yhi


def up_tolerance(Yu):
    """The product tolerance band of the up layer: 8e-3 |Y| + 1e-3 rms(Y)."""
    return 8e-3 * np.abs(Yu) + 1e-3 * np.sqrt(np.mean(Yu ** 2))
