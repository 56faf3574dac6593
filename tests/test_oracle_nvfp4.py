"""Pins for the oracle's NVFP4 encoding.

The pages name NVFP4 ("Optimizing FLUX 3 Image Klein inference on NVIDIA
Blackwell GPUs", How it works) without defining it; the reading is stated in
``oracle.nvfp4``.  These tests pin the implementation of that reading to
things other than itself: an independent re-encoding with library codecs,
exact closed forms, and invariants.
"""

import ml_dtypes
import numpy as np
import pytest

from oracle import codecs, nvfp4
from synth import normal_bf16


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _library_encode(x):
    """Same reading, but every rounding done by ml_dtypes and the loops
    written per block (independent of the vectorised oracle)."""
    x = _f32(x)
    R, C = x.shape
    amax = np.float32(np.abs(x).max())
    gs = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2688.0))
    inv = np.float32(np.float32(1.0) / np.float32(np.float32(6.0) * gs))
    codes = np.zeros((R, C), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    for r in range(R):
        for b in range(C // 16):
            blk = x[r, 16 * b:16 * b + 16]
            ab = np.float32(np.abs(blk).max())
            if ab == 0:
                continue
            sv = np.float32(ab * inv)
            sb = np.array([min(sv, np.float32(448.0))], np.float32).astype(ml_dtypes.float8_e4m3fn)
            scales[r, b] = sb.view(np.uint8)[0]
            S = np.float32(np.float32(sb.astype(np.float32)[0]) * gs)
            if S == 0:
                continue
            rr = np.float32(np.float32(1.0) / S)
            y = (blk * rr).astype(np.float32)
            codes[r, 16 * b:16 * b + 16] = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    packed = codes[:, 0::2] | (codes[:, 1::2] << 4)
    return packed, scales, gs


@pytest.mark.parametrize("shape,seed,std", [((8, 64), 0, 1.0), ((5, 48), 1, 0.02), ((3, 256), 2, 30.0)])
def test_matches_library_encoding(shape, seed, std):
    x = normal_bf16(shape, seed, std).float().numpy()
    c, s, g = nvfp4.quantize(x)
    c2, s2, g2 = _library_encode(x)
    assert g == g2
    np.testing.assert_array_equal(s, s2)
    np.testing.assert_array_equal(c, c2)


def test_exact_ties_closed_form():
    # Tensor amax 2.625 = 2688 * 2^-10, so gs = 2^-10 exactly.  Block 1 has
    # amax 1.5 = 6 * 256 * 2^-10, so amax_b * inv = 256 * (1 + O(2^-24)) and the
    # E4M3 scale is exactly 256 (code 0x78); S = 2^-2 and r = 4 are exact, so
    # block 1's codes are E2M1 of exact multiples of 0.25 -- the midpoints
    # 0.25, 0.75, ... land on exact ties and must go to the even code.
    blk0 = np.zeros(16, np.float32)
    blk0[0] = 2.625
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0,
                     -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.0], np.float32)
    blk1 = mids * np.float32(0.25)
    x = np.concatenate([blk0, blk1])[None, :]
    codes, scales, gs = nvfp4.quantize(x)
    assert gs == np.float32(2.0**-10)
    assert scales[0, 1] == 0x78 and codecs.e4m3_decode(0x78) == 256.0
    assert scales[0, 0] == 0x7E                      # 2.625 / (6 gs) = 448
    want = np.array([0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x7,
                     0x8, 0xA, 0xA, 0xC, 0xC, 0xE, 0xE, 0x0], np.uint8)
    got = nvfp4.unpack_codes(codes)[0, 16:]
    np.testing.assert_array_equal(got, want)
    # packing: element 2i in the low nibble
    assert codes[0, 8] == (want[0] | (want[1] << 4))


def test_zero_tensor_and_zero_blocks():
    x = np.zeros((2, 32), np.float32)
    c, s, g = nvfp4.quantize(x)
    assert g == 1.0 and not c.any() and not s.any()
    x[1, 20] = -3.0
    c, s, g = nvfp4.quantize(x)
    assert s[0].sum() == 0 and s[1, 0] == 0 and s[1, 1] != 0
    d = nvfp4.dequantize(c, s, g)
    assert d[1, 20] == pytest.approx(-3.0, rel=2**-3)
    assert np.count_nonzero(d) == 1


def test_single_element_and_amax_element_exact():
    # a block holding one value v: sb ~ v / (6 gs) and the code is +-6, so
    # the decoded value is within E4M3's half-ulp (2^-4) of v
    x = np.zeros((1, 16), np.float32)
    x[0, 5] = -1.171875
    c, s, g = nvfp4.quantize(x)
    assert nvfp4.unpack_codes(c)[0, 5] == 0xF     # -6
    assert abs(nvfp4.dequantize(c, s, g)[0, 5] / -1.171875 - 1) <= 2**-4


def test_invariants_random():
    x = normal_bf16((64, 512), 11, 1.0).float().numpy()
    c, s, g = nvfp4.quantize(x)
    codes = nvfp4.unpack_codes(c)
    vals = codecs.e2m1_decode(codes)
    assert set(np.abs(vals).ravel()).issubset({0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0})
    S = codecs.e4m3_decode(s) * np.float64(g)                       # [R, C/16]
    amax_t = np.abs(x).max()
    # the largest block scale reaches the tensor amax (E4M3 rounding <= 2^-4)
    assert (S * 6).max() >= amax_t * (1 - 2**-3)
    # reconstruction error within half an E2M1 gap (scaled), below the clamp
    dec = nvfp4.dequantize(c, s, g)
    Sx = np.repeat(S, 16, axis=1)
    mag = np.abs(x) / Sx
    gap = np.select([mag < 2, mag < 4], [0.5, 1.0], 2.0)
    ok = mag <= 6
    assert np.all(np.abs(x - dec)[ok] <= (gap / 2 * Sx)[ok] * (1 + 1e-6))


def test_reencode_fixed_point():
    # values that are exactly code * S, with one +-6 per block, re-encode to
    # the same codes and scales when the same global scale is used
    rng = np.random.default_rng(5)
    R, C = 4, 64
    codes = rng.integers(0, 16, size=(R, C)).astype(np.uint8)
    codes[:, ::16] = 7                                     # a +6 in every block
    sb = rng.integers(0x20, 0x70, size=(R, C // 16)).astype(np.uint8)
    gs = np.float32(2.0**-7)
    vals = codecs.e2m1_decode(codes) * np.repeat(codecs.e4m3_decode(sb), 16, axis=1) * np.float64(gs)
    c2, s2, _ = nvfp4.quantize(vals.astype(np.float32), gs=gs)
    np.testing.assert_array_equal(s2, sb)
    np.testing.assert_array_equal(nvfp4.unpack_codes(c2)[codes != 8], codes[codes != 8])


def test_block_scale_extremes():
    # a block 2^-120 times smaller than the rest rounds its scale towards the
    # E4M3 subnormal floor or zero; a huge tensor keeps a finite gs
    x = normal_bf16((2, 64), 3, 1.0).float().numpy()
    x[1, 16:32] *= np.float32(2.0**-120)
    c, s, g = nvfp4.quantize(x)
    assert s[1, 1] == 0 or codecs.e4m3_decode(s[1, 1]) <= 2.0**-9
    y = x * np.float32(2.0**100)
    c, s, g = nvfp4.quantize(y)
    assert np.isfinite(g) and g > 0
    assert (codecs.e4m3_decode(s) * g * 6).max() >= np.abs(y).max() * (1 - 2**-3)
