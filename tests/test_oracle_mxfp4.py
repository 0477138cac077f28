"""Pins for the oracle's MXFP4 encoder (no GPU).

What fixes the expected values here is not the oracle itself:
* hand-worked block encodings in tests/golden/mxfp4_hand_vectors.txt;
* the E2M1 grid of the OCP MX format (every grid value encodes to itself,
  every midpoint goes to the even code, values beyond 6 saturate);
* the invariant of the shared exponent (the block maximum lands in [4, 8));
* brute-force element-by-element dequantisation on tiny inputs.
"""
import os

import numpy as np
import pytest

from oracle import w4a4_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_hand_vectors.txt")


def _parse_float(tok):
    tok = tok.strip()
    if "0x" in tok or "0X" in tok:
        return np.float32(float.fromhex(tok))
    return np.float32(tok)


def _load_golden():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, vals, sc, codes = [p.strip() for p in line.split("|")]
        v = np.zeros(32, np.float32)
        vv = [_parse_float(t) for t in vals.split(",")]
        v[:len(vv)] = vv
        c = np.zeros(32, np.uint8)
        cc = [int(t, 16) for t in codes.split(",")]
        c[:len(cc)] = cc
        cases.append((name, v, int(sc), c, len(vv)))
    return cases


@pytest.mark.parametrize("case", _load_golden(), ids=lambda c: c[0])
def test_hand_vectors(case):
    name, v, sc, codes, n = case
    got_sc, got_codes = orc.mxfp4_quantize_blocks(v[None, :])
    assert int(got_sc[0]) == sc, name
    np.testing.assert_array_equal(got_codes[0, :n], codes[:n], err_msg=name)
    # unlisted elements are +0 -> code 0, except where the row is all -0 (H lists them)
    np.testing.assert_array_equal(got_codes[0, n:], np.zeros(32 - n, np.uint8), err_msg=name)


def test_grid_values_encode_to_themselves():
    grid = orc.E2M1_GRID.astype(np.float32)
    for sign in (1.0, -1.0):
        q = (sign * grid).astype(np.float32)
        codes = orc.e2m1_codes(q)
        np.testing.assert_array_equal(codes & 7, np.arange(8))
        back = orc.e2m1_value(codes)
        np.testing.assert_array_equal(back, sign * orc.E2M1_GRID)


def test_midpoints_round_to_even_and_saturate():
    g = orc.E2M1_GRID
    mids = (g[:-1] + g[1:]) / 2
    codes = orc.e2m1_codes(mids.astype(np.float32)) & 7
    # the even code of the two neighbours
    lo = np.arange(7)
    expect = np.where(lo % 2 == 0, lo, lo + 1)
    np.testing.assert_array_equal(codes, expect)
    big = np.array([6.0, 6.5, 7.999, 1e30, np.float32(3.4e38)], np.float32)
    np.testing.assert_array_equal(orc.e2m1_codes(big) & 7, 7)


def test_rounding_is_nearest_by_brute_force():
    rng = np.random.default_rng(3)
    q = rng.uniform(-8, 8, 20000).astype(np.float32)
    codes = orc.e2m1_codes(q)
    val = orc.e2m1_value(codes)
    err = np.abs(val - np.clip(q.astype(np.float64), -6, 6))
    # distance to every grid point (with sign) must be >= the chosen distance
    grid = np.concatenate([-orc.E2M1_GRID, orc.E2M1_GRID])
    dmin = np.min(np.abs(np.clip(q, -6, 6)[:, None].astype(np.float64) - grid[None, :]), axis=1)
    np.testing.assert_allclose(err, dmin, rtol=0, atol=0)


def test_block_maximum_lands_in_top_binade():
    rng = np.random.default_rng(5)
    for scale in (1e-30, 1e-5, 0.3, 1.0, 17.0, 1e20):
        V = (rng.standard_t(3, size=(200, 32)) * scale).astype(np.float32)
        sc, codes = orc.mxfp4_quantize_blocks(V)
        e = sc.astype(np.int64) - 127
        amax = np.max(np.abs(V), axis=1)
        ok = e > -127
        qmax = np.ldexp(amax.astype(np.float64), -e)
        assert np.all((qmax[ok] >= 4) & (qmax[ok] < 8))
        # the element holding the maximum is coded 4 or 6 (magnitude nibble 6 or 7)
        imax = np.argmax(np.abs(V), axis=1)
        top = codes[np.arange(200), imax] & 7
        assert np.all(np.isin(top[ok], (6, 7)))


def test_dequant_by_elementwise_definition():
    rng = np.random.default_rng(11)
    V = (rng.normal(size=(3, 64)) * np.array([[0.01], [1.0], [300.0]])).astype(np.float32)
    blocks = V.reshape(3, 2, 32)
    sc, codes = orc.mxfp4_quantize_blocks(blocks)
    packed = orc.pack_nibbles(codes.reshape(3, 64))
    deq = orc.dequant_mxfp4(packed, sc)
    table = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}
    for r in range(3):
        for j in range(64):
            byte = int(packed[r, j // 2])
            nib = (byte >> 4) if j % 2 else (byte & 0xF)
            mag = table[nib & 7]
            val = (-mag if nib & 8 else mag) * 2.0 ** (int(sc[r, j // 32]) - 127)
            assert deq[r, j] == val
            # quantisation error bounded by half the local grid spacing times the scale
            q = abs(float(V[r, j])) * 2.0 ** -(int(sc[r, j // 32]) - 127)
            half = 0.25 if q < 2 else (0.5 if q < 4 else (1.0 if q <= 6 else q - 6))
            assert abs(val - float(V[r, j])) <= half * 2.0 ** (int(sc[r, j // 32]) - 127)


def test_nibble_order():
    codes = np.array([[1, 2, 3, 4]], np.uint8)
    np.testing.assert_array_equal(orc.pack_nibbles(codes), [[0x21, 0x43]])
    np.testing.assert_array_equal(orc.unpack_nibbles(orc.pack_nibbles(codes)), codes)


def test_bf16_rounding_definition():
    # exact bf16 values round-trip; halfway cases go to the even mantissa
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-7, -2.5, 3.4e38], np.float32)
    bits = orc.f32_to_bf16_bits(x)
    back = orc.bf16_bits_to_f32(bits)
    np.testing.assert_array_equal(back[[0, 3, 4]], x[[0, 3, 4]])
    assert back[1] == 1.0                      # halfway -> even (1.0)
    assert back[2] == 1.0 + 2 * 2**-7          # halfway -> even (1 + 2^-6)
    assert np.isinf(back[5])                   # 3.4e38 is past the halfway point above the bf16 maximum
    # compare against torch's conversion on random data
    import torch
    r = np.random.default_rng(0).normal(size=10000).astype(np.float32) * 100
    tb = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.f32_to_bf16_bits(r), tb)


def test_mma_scale_layout_is_a_bijection():
    rows, nblk = 256, 8
    offs = {orc.mma_sf_offset(r, kb, nblk) for r in range(rows) for kb in range(nblk)}
    assert offs == set(range(rows * nblk))
    # atom structure: 4 consecutive blocks of one row are 4 consecutive bytes
    assert [orc.mma_sf_offset(5, kb, nblk) for kb in range(4)] == [80, 81, 82, 83]
    # rows 32 apart inside a 128-row atom sit 4 bytes apart
    assert orc.mma_sf_offset(37, 0, nblk) - orc.mma_sf_offset(5, 0, nblk) == 4
    # the second K atom of row-block 0 starts at byte 512, row-block 1 after all K atoms
    assert orc.mma_sf_offset(0, 4, nblk) == 512
    assert orc.mma_sf_offset(128, 0, nblk) == 1024


def test_dequant_of_the_non_finite_scale_codes():
    # E8M0: code 254 is 2^127, the largest scale; 0xFF is NaN and makes its
    # whole block NaN, whatever the element codes (here all zero)
    codes = np.zeros((2, 32), np.uint8)
    codes[0, :3] = [0x7, 0xF, 0x2]                    # 6, -6, 1
    sf = np.array([[254], [255]], np.uint8)
    deq = orc.dequant_mxfp4(orc.pack_nibbles(codes), sf)
    assert deq[0, 0] == 6.0 * 2.0 ** 127 and deq[0, 1] == -6.0 * 2.0 ** 127
    assert deq[0, 2] == 2.0 ** 127 and deq[0, 3] == 0.0
    assert np.isnan(deq[1]).all()


def test_nan_and_inf_blocks_among_finite_ones():
    # a row of three blocks: finite, holding an infinity, holding a NaN --
    # each block is coded on its own, the finite one exactly as if alone
    rng = np.random.default_rng(2)
    V = rng.normal(size=(1, 3, 32)).astype(np.float32)
    alone_sc, alone_codes = orc.mxfp4_quantize_blocks(V[:, 0])
    V[0, 1, 7] = -np.inf
    V[0, 2, 30] = np.nan
    sc, codes = orc.mxfp4_quantize_blocks(V)
    assert sc[0, 0] == alone_sc[0] and (codes[0, 0] == alone_codes[0]).all()
    assert sc[0, 1] == 254 and codes[0, 1, 7] == 0xF
    # the block's finite normals, scaled by 2^-127, all lie below 0.25
    assert ((codes[0, 1, np.arange(32) != 7] & 7) == 0).all()
    assert sc[0, 2] == 255 and not codes[0, 2].any()
