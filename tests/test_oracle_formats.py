"""Pins for the oracle's element formats and global scale (CPU only).

The E2M1 and E4M3 encoders are checked against hand-worked tables derived from
the format definitions (tests/golden), against an independent library
(ml_dtypes), and exhaustively (every code round-trips, every midpoint goes to
the even code).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from conftest import read_golden


def test_e2m1_hand_table():
    for v, code in read_golden("e2m1_rne.txt"):
        assert O.e2m1_encode(np.float32(v)) == int(code, 16), v


def test_e4m3_hand_table():
    for v, code in read_golden("e4m3_rne.txt"):
        assert O.e4m3_encode(np.float32(v)) == int(code, 16), v


def test_e2m1_decode_all_codes_vs_ml_dtypes():
    for c in range(16):
        lib = float(np.array([c], np.uint8).view(ml_dtypes.float4_e2m1fn)[0])
        got = O.e2m1_decode(c)
        assert got == lib and np.signbit(got) == np.signbit(lib), c


def test_e4m3_decode_all_codes_vs_ml_dtypes():
    for b in range(256):
        lib = float(np.array([b], np.uint8).view(ml_dtypes.float8_e4m3fn)[0])
        got = O.e4m3_decode(b)
        if np.isnan(lib):
            assert np.isnan(got), b
        else:
            assert got == lib, b


def test_e2m1_encode_matches_ml_dtypes_sweep():
    rng = np.random.default_rng(123)
    vals = np.concatenate([
        rng.uniform(-8, 8, 20000).astype(np.float32),
        rng.normal(0, 1, 5000).astype(np.float32),
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0], np.float32),
    ])
    lib = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    for v, want in zip(vals, lib):
        assert O.e2m1_encode(v) == int(want), v


def test_e4m3_encode_matches_ml_dtypes_in_range():
    # Inside [0, 464] round-to-nearest-even and the saturating variant agree,
    # so the library conversion is a reference there.
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.uniform(0, 464, 4000), np.exp(rng.uniform(np.log(1e-4), np.log(460), 4000)),
        rng.uniform(0, 0.02, 2000)]).astype(np.float32)
    lib = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    for v, want in zip(vals, lib):
        assert O.e4m3_encode(v) == int(want), v


def test_e4m3_exhaustive_roundtrip_and_midpoints():
    finite = [b for b in range(0x7F)]
    vals = [O.e4m3_decode(b) for b in finite]
    assert vals == sorted(vals) and len(set(vals)) == len(vals)
    for b, v in zip(finite, vals):
        assert O.e4m3_encode(np.float32(v)) == b
    for b in range(0x7E):
        lo, hi = vals[b], vals[b + 1]
        mid = np.float32((np.float64(lo) + np.float64(hi)) / 2)
        assert float(mid) == (lo + hi) / 2            # midpoints are exact in fp32
        want = b if b % 2 == 0 else b + 1
        assert O.e4m3_encode(mid) == want
        assert O.e4m3_encode(np.nextafter(mid, np.float32(0))) == b
        assert O.e4m3_encode(np.nextafter(mid, np.float32(1e9))) == b + 1
    for big in [448.0, 449.0, 1e6, 3.0e38]:
        assert O.e4m3_encode(np.float32(big)) == 0x7E
    assert O.e4m3_encode(np.float32(-2.0)) == 0x80 | O.e4m3_encode(np.float32(2.0))


def test_e2m1_exhaustive_roundtrip_and_midpoints():
    mags = [O.e2m1_decode(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        assert O.e2m1_encode(np.float32(O.e2m1_decode(c))) == c
    for c in range(7):
        mid = np.float32((mags[c] + mags[c + 1]) / 2)
        want = c if c % 2 == 0 else c + 1
        assert O.e2m1_encode(mid) == want
        assert O.e2m1_encode(-mid) == 8 | want


@pytest.mark.parametrize("amax,gs", [(2688.0, 1.0), (1.0, 2688.0), (0.0, 1.0), (2.0, 1344.0),
                                     (1.0 / 1024, 2688.0 * 1024)])
def test_global_scale_closed_forms(amax, gs):
    assert O.global_scale_from_amax(np.float32(amax)) == np.float32(gs)


def test_global_scale_inverts_amax():
    rng = np.random.default_rng(3)
    for a in np.exp(rng.uniform(-20, 20, 200)).astype(np.float32):
        gs = O.global_scale_from_amax(a)
        # gs is 2688/amax rounded once: |gs*amax - 2688| <= 2688 * 2^-24 (+ the product's rounding)
        assert abs(np.float64(gs) * np.float64(a) - 2688.0) <= 2688.0 * 2.0 ** -23


def test_amax_bf16_and_f32():
    x = np.array([0.5, -3.25, 2.0, -0.0], np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert O.amax_bf16(bits) == np.float32(3.25)
    assert O.amax_f32(x) == np.float32(3.25)
    assert O.amax_f32(np.zeros(5, np.float32)) == 0.0
