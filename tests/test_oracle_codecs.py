"""Pins for the oracle's narrow-float codecs against independent library codecs.

ml_dtypes (float8_e4m3fn, float4_e2m1fn) and torch.float8_e4m3fn are separate
implementations of the same OCP formats; torch's fp32 -> bf16 cast is a
separate implementation of bf16 round-to-nearest-even.
"""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import codecs

E2M1_SET = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}


def _sweep(lo, hi, n, seed=0):
    rng = np.random.default_rng(seed)
    dense = np.linspace(lo, hi, n, dtype=np.float64).astype(np.float32)
    rand = rng.uniform(lo, hi, n).astype(np.float32)
    return np.concatenate([dense, rand])


def _with_neighbours(vals):
    v = np.asarray(vals, dtype=np.float32)
    up = np.nextafter(v, np.float32(np.inf))
    dn = np.nextafter(v, np.float32(-np.inf))
    return np.concatenate([v, up, dn, -v, -up, -dn])


def test_e2m1_value_set():
    # every one of the 16 codes decodes into {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}
    vals = codecs.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert {abs(float(v)) for v in vals} == E2M1_SET
    assert len(set(float(v) for v in vals)) == 15  # +0 and -0 compare equal


def test_e2m1_encode_matches_ml_dtypes():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    grid = np.array(sorted(E2M1_SET), dtype=np.float32)
    x = np.concatenate([_sweep(-8, 8, 20001), _with_neighbours(mids), _with_neighbours(grid),
                        np.array([7.0, -7.0, 100.0, -1e30, 1e-30, -1e-30, 0.0, -0.0], np.float32)])
    ours = codecs.e2m1_encode(x)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(ours, ref)
    # only the 16 codes come out, and they decode into the value set
    assert set(np.unique(ours)).issubset(set(range(16)))


def test_e2m1_ties_to_even():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    want = np.array([0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0])
    np.testing.assert_array_equal(codecs.e2m1_decode(codecs.e2m1_encode(mids)), want)
    # a negative value that rounds to zero keeps its sign bit
    assert codecs.e2m1_encode(np.float32(-0.1)) == 0x8


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])
    tref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours[ok], tref[ok])
    assert codecs.E4M3_MAX == 448.0 and ours[0x7E] == 448.0


def test_e4m3_encode_matches_libraries():
    finite = codecs.E4M3_FINITE.astype(np.float32)
    mids = ((codecs.E4M3_FINITE[1:] + codecs.E4M3_FINITE[:-1]) / 2).astype(np.float32)
    x = np.concatenate([_sweep(-500, 500, 40001), _sweep(-1, 1, 20001, 1), _sweep(-0.02, 0.02, 20001, 2),
                        _with_neighbours(finite), _with_neighbours(mids),
                        np.array([2.0**-10, 2.0**-11, 1e-30, 460.0, 464.0, 1e9, -1e9], np.float32)])
    ours = codecs.e4m3_encode(x)
    clamped = np.clip(x, -448.0, 448.0)
    ref = clamped.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(ours, ref)
    tref = torch.from_numpy(clamped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, tref)
    # saturation of infinities, NaN code
    assert codecs.e4m3_encode(np.float32(np.inf)) == 0x7E
    assert codecs.e4m3_encode(np.float32(-np.inf)) == 0xFE
    assert codecs.e4m3_encode(np.float32(np.nan)) == 0x7F


def test_bf16_round_matches_torch_on_fp32():
    rng = np.random.default_rng(3)
    x = np.concatenate([(rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000)).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1 + 2**-8, 1 + 2**-9, 1 + 3 * 2**-9, 2.0**-130, 3e38], np.float32)])
    assert x.dtype == np.float32
    ours = codecs.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_bf16_round_fp64_is_nearest():
    # one rounding straight from fp64: the result is the nearer of the two
    # neighbouring bf16 values (ties to the even mantissa)
    rng = np.random.default_rng(4)
    x = rng.standard_normal(20000) * 10.0 ** rng.integers(-5, 5, 20000)
    r = codecs.bf16_round(x).astype(np.float64)
    bits = codecs.bf16_bits(codecs.bf16_round(x))
    up = codecs.bf16_from_bits(bits + 1).astype(np.float64)
    dn = codecs.bf16_from_bits(bits - 1).astype(np.float64)
    err = np.abs(x - r)
    assert np.all(err <= np.abs(x - up)) and np.all(err <= np.abs(x - dn))
    # exact ties go to the even mantissa
    t = np.array([1 + 2**-8, 1 + 3 * 2**-8], np.float64)
    np.testing.assert_array_equal(codecs.bf16_round(t), np.array([1.0, 1 + 2**-6], np.float32))


@pytest.mark.parametrize("v", [0.3, -2.7, 1e-3])
def test_bf16_bits_roundtrip(v):
    b = codecs.bf16_round(np.float64(v))
    assert codecs.bf16_from_bits(codecs.bf16_bits(b)) == b
