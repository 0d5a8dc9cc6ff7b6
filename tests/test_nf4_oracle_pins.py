"""Pins for the NF4 oracle (oracle/nf4_ref.py):
* the 16 levels against the same quantile definition evaluated another way
  (bisection on math.erf instead of scipy's inverse normal CDF), and their
  shape: ascending, exact zero at code 7, -1 and 1 at the ends, 7 negative and
  8 positive levels;
* the post's 0.37 bit per parameter saved by double quantization
  (tests/golden/double_quant_bits.json);
* quantize / dequantize: weights that are levels times a block scale come
  back up to the scale's 8-bit rounding; random weights within half the
  largest level gap; codes are nearest levels;
* the projection's q, k, v are the row blocks of x W^T.
"""
import json
import math
import os

import numpy as np

import oracle.nf4_ref as nr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _phi_inv(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * (1.0 + math.erf(mid / math.sqrt(2.0))) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_levels_against_bisection_and_shape():
    lv = nr.nf4_levels()
    top = _phi_inv(1 - nr.NF4_DELTA)
    pos = [_phi_inv(p) / top for p in np.linspace(0.5, 1 - nr.NF4_DELTA, 9)]
    neg = [-_phi_inv(p) / top for p in np.linspace(0.5, 1 - nr.NF4_DELTA, 8)[1:]]
    np.testing.assert_allclose(lv, np.sort(pos + neg), atol=1e-12, rtol=0)
    assert lv.shape == (16,) and np.all(np.diff(lv) > 0)
    assert lv[7] == 0.0 and lv[0] == -1.0 and lv[15] == 1.0
    assert (lv < 0).sum() == 7 and (lv > 0).sum() == 8


def test_double_quant_saves_the_posts_bits():
    gd = json.load(open(os.path.join(GOLDEN, "double_quant_bits.json")))
    saved = nr.bits_per_weight(False) - nr.bits_per_weight(True)
    assert abs(saved - gd["saved_bits_per_parameter"]) < gd["tolerance"]


def test_round_trip():
    rng = np.random.default_rng(1)
    lv = nr.nf4_levels()
    rows, K = 8, 2048                                    # 256 first-level blocks: one second-level block
    scales = rng.uniform(0.01, 0.05, size=rows * K // 64)
    codes_in = rng.integers(0, 16, size=(rows * K // 64, 64))
    codes_in[:, 0] = 15                                  # every block reaches its absmax
    w = (lv[codes_in] * scales[:, None]).reshape(rows, K)
    codes, sq, c2 = nr.quantize_nf4(w)
    np.testing.assert_array_equal(codes.reshape(-1, 64), codes_in)
    wd = nr.dequantize_nf4(codes, sq, c2)
    # only the 8-bit scale rounding remains: |w' - w| <= |w| * (c2 / 127 / 2) / scale
    err = np.abs(wd - w).reshape(-1, 64).max(axis=1)
    assert np.all(err <= scales * 0 + c2.max() / 127 / 2 + 1e-15)
    # random weights: within half the largest gap times the block scale (plus the scale rounding)
    w2 = rng.standard_normal((16, 1024)) * 0.02
    c, s, cc = nr.quantize_nf4(w2)
    wd2 = nr.dequantize_nf4(c, s, cc)
    absmax = np.abs(w2.reshape(-1, 64)).max(axis=1)
    bound = absmax * (np.diff(lv).max() / 2) + cc.max() / 127 / 2
    assert np.all(np.abs(wd2 - w2).reshape(-1, 64).max(axis=1) <= bound + 1e-15)
    # codes are nearest levels of w / absmax
    x = w2.reshape(-1, 64) / absmax[:, None]
    assert np.all(np.abs(x - lv[c.reshape(-1, 64)]) <= np.abs(x[..., None] - lv).min(-1) + 1e-15)


def test_partial_last_second_level_block():
    """48 first-level blocks: one second-level block of 48 (ceil(48 / 256) = 1);
    weights that are levels times a scale still come back up to the 8-bit
    scale rounding, and the second-level scale is the largest absmax."""
    rng = np.random.default_rng(3)
    lv = nr.nf4_levels()
    rows, K = 3, 1024
    scales = rng.uniform(0.01, 0.05, size=rows * K // 64)
    codes_in = rng.integers(0, 16, size=(rows * K // 64, 64))
    codes_in[:, 0] = 0                                   # level -1: absmax = scale
    w = (lv[codes_in] * scales[:, None]).reshape(rows, K)
    codes, sq, c2 = nr.quantize_nf4(w)
    assert c2.shape == (1,) and abs(float(c2[0]) - scales.max()) <= 2 ** -24 * scales.max()  # stored as float32
    np.testing.assert_array_equal(codes.reshape(-1, 64), codes_in)
    err = np.abs(nr.dequantize_nf4(codes, sq, c2) - w).max()
    assert err <= float(c2[0]) / 127 / 2 + 1e-12


def test_projection_row_blocks():
    rng = np.random.default_rng(2)
    B, N, dm, H, Hkv, D = 1, 8, 256, 4, 2, 32
    w = rng.standard_normal(((H + 2 * Hkv) * D, dm)) * 0.02
    codes, sq, c2 = nr.quantize_nf4(w)
    x = rng.standard_normal((B, N, dm))
    q, k, v = nr.nf4_qkv_projection(x, codes, sq, c2, H, Hkv, D)
    wd = nr.dequantize_nf4(codes, sq, c2)
    np.testing.assert_allclose(q[0, 3, 1], x[0, 3] @ wd[D:2 * D].T, atol=1e-12, rtol=0)
    np.testing.assert_allclose(k[0, 5, 1], x[0, 5] @ wd[(H + 1) * D:(H + 2) * D].T, atol=1e-12, rtol=0)
    np.testing.assert_allclose(v[0, 7, 0], x[0, 7] @ wd[(H + Hkv) * D:(H + Hkv + 1) * D].T, atol=1e-12, rtol=0)


def test_bf16_operand_reading():
    """dequantize_nf4_bf16: within one bf16 ulp of the exact dequantized value
    everywhere, equal to its nearest bf16 almost everywhere (the float32 steps
    decide only near-ties), and bit-exact against a hand evaluation of the
    float32 steps for a few entries (Python floats through struct)."""
    import struct

    def f32(v):
        return struct.unpack("f", struct.pack("f", v))[0]

    rng = np.random.default_rng(9)
    rows, K = 16, 4096
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    nblk = rows * K // 64
    sq = rng.integers(64, 128, size=nblk).astype(np.int8)
    c2 = rng.uniform(0.05, 0.08, size=(nblk + 255) // 256).astype(np.float32)
    exact = nr.dequantize_nf4(codes, sq, c2)
    w = nr.dequantize_nf4_bf16(codes, sq, c2)
    rn = nr.round_bf16(exact)
    assert np.all(np.abs(w - exact) <= np.abs(rn) * 2.0 ** -7)
    assert np.mean(w == rn) >= 0.999
    lv = nr.nf4_levels()
    for (r, k) in [(0, 0), (3, 777), (15, 4095)]:
        blk = (r * K + k) // 64
        s = f32(f32(float(sq[blk]) * float(c2[blk // 256])) / 127.0)
        v = f32(f32(float(lv[codes[r, k]])) * s)
        assert w[r, k] == float(nr.round_bf16(np.array([v]))[0])
