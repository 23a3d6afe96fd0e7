"""Pins for the oracle's block quantiser and dequantiser (CPU only)."""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from conftest import read_golden


def f32_to_bf16_bits(x):
    """Round-to-nearest-even fp32 -> bf16 bit patterns (numpy only)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def unpack_codes(codes):
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


E2M1_VALUE = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def e4m3_value(b):
    return np.asarray(b, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_worked_block():
    rows = {r[0]: r[1:] for r in read_golden("worked_block.txt")}
    gs = float(rows["gs"][0])
    x = np.array([float(v) for v in rows["x"]], np.float32)[None, :]
    codes, scales = O.quantize_f32(x, gs)
    assert scales[0, 0] == int(rows["scale"][0], 16)
    want = [int(v, 16) for v in rows["q"]]
    assert unpack_codes(codes)[0].tolist() == want
    # nibble order: element 2i in the low nibble of byte i
    assert codes[0, 0] == (want[0] | (want[1] << 4))


def _random_blocks(rng, rows, cols):
    x = rng.normal(0, 1, (rows, cols)).astype(np.float32)
    x *= np.exp(rng.uniform(-6, 6, (rows, 1))).astype(np.float32)   # per-row magnitude spread
    x[0, :16] = 0.0                                                  # an all-zero block
    return x


def test_invariants_against_independent_rounding():
    """For every block: s == E4M3(amax/6*gs) and q_i == E2M1(x_i*gs/s), with the
    format rounding done by ml_dtypes and the fp32 steps by numpy."""
    rng = np.random.default_rng(11)
    x = _random_blocks(rng, 64, 256)
    gs = O.global_scale_from_amax(np.abs(x).max())
    codes, scales = O.quantize_f32(x, gs)
    blocks = x.reshape(-1, 16)
    amax = np.abs(blocks).max(axis=1).astype(np.float32)
    v = (amax / np.float32(6.0)).astype(np.float32) * np.float32(gs)
    s_ref = v.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(scales.reshape(-1), s_ref)
    sval = e4m3_value(s_ref).astype(np.float32)
    r = np.where(sval == 0, np.float32(0), np.float32(gs) / np.where(sval == 0, 1, sval)).astype(np.float32)
    q_ref = (blocks * r[:, None]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    assert np.array_equal(unpack_codes(codes).reshape(-1, 16), q_ref)


def test_bounds_and_error():
    rng = np.random.default_rng(5)
    x = _random_blocks(rng, 32, 512)
    gs = O.global_scale_from_amax(np.abs(x).max())
    codes, scales = O.quantize_f32(x, gs)
    q = unpack_codes(codes)
    assert np.all(np.abs(E2M1_VALUE[q]) <= 6.0)
    assert not np.any(scales == 0x7F) and not np.any(scales == 0xFF)
    dq = O.dequantize(codes, scales, gs).astype(np.float64)
    assert np.all(np.isfinite(dq))
    s = np.repeat(e4m3_value(scales), 16, axis=1)
    # |dq - x| <= half the E2M1 spacing at |x*r| times s/gs; where s rounded
    # below amax/6*gs, |x*r| may pass 6 and the element clips to 6 instead.
    scaled = np.abs(x.astype(np.float64)) * np.where(s > 0, gs / np.where(s > 0, s, 1), 0)
    spacing = np.where(scaled < 2, 0.5, np.where(scaled < 4, 1.0, 2.0))
    half = np.where(scaled <= 6, 0.5 * spacing, scaled - 6)
    normal = s >= 2.0 ** -6                            # E4M3 normal range: rounds down by < 1/16
    assert np.all(scaled[normal] <= 6 * 16 / 15 + 1e-6)
    err = np.abs(dq - x)
    bound = half * s / gs * (1 + 1e-6) + np.abs(dq) * 2.0 ** -23   # + dq's own fp32 rounding
    nz = s > 0
    assert np.all(err[nz] <= bound[nz])
    # blocks whose scale underflowed to 0 dequantise to 0
    assert np.all(dq[~nz] == 0)


def test_zero_and_underflow_blocks():
    """A zero block gives s = 0 and zero codes.  With gs = 2688 (tensor amax 1)
    the block scale underflows to 0 exactly when amax/6*gs < 2^-10, i.e. for a
    block amax below about 2.18e-6; just above, it is the smallest subnormal."""
    x = np.zeros((1, 48), np.float32)
    x[0, 16:32] = 2.0e-6 * np.linspace(-1, 1, 16)
    x[0, 32:48] = 2.3e-6 * np.linspace(-1, 1, 16)
    gs = O.global_scale_from_amax(1.0)
    codes, scales = O.quantize_f32(x, gs)
    assert scales.tolist() == [[0, 0, 1]]
    q = unpack_codes(codes)[0]
    assert set(q[:16].tolist()) == {0}
    assert set(q[16:32].tolist()) <= {0, 8}            # zero or negative zero


def test_oversized_global_scale_saturates_without_nan():
    """The pages' failure: a multiplier of 3977.6 against activations of amax
    about 1.27 ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 2, "What the quant
    method does").  With saturating conversion the block scale clamps to 448
    and no NaN appears."""
    rng = np.random.default_rng(0)
    x = rng.uniform(-1.27, 1.27, (4, 64)).astype(np.float32)
    x[0, 0] = 1.27
    gs = np.float32(3977.6)
    codes, scales = O.quantize_f32(x, gs)
    assert scales[0, 0] == 0x7E                     # 1.27/6*3977.6 = 841.9 -> 448
    dq = O.dequantize(codes, scales, gs)
    assert np.all(np.isfinite(dq))
    assert np.all(np.abs(unpack_codes(codes).astype(int) & 7) <= 7)


def test_no_nan_for_any_gs_up_to_limit():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 3, (8, 128)).astype(np.float32)
    amax = np.abs(x).max()
    for gs in [O.global_scale_from_amax(amax), np.float32(1e-3), np.float32(1.0), np.float32(1e6)]:
        codes, scales = O.quantize_f32(x, gs)
        assert not np.any((scales & 0x7F) == 0x7F)
        assert np.all(np.isfinite(O.dequantize(codes, scales, gs)))


def test_representable_values_roundtrip_exactly():
    """x = v * s / gs with v an E2M1 value and s = the block's E4M3 scale
    (chosen so that amax maps exactly to 6) must dequantise back exactly."""
    gs = np.float32(64.0)
    s = np.float32(2.0)                               # amax = 6*s/gs = 0.1875
    v = np.array([6, -6, 4, 3, -2, 1.5, 1, .5, 0, -.5, 6, 2, -3, 4, -1, 1.5], np.float32)
    x = (v * s / gs).astype(np.float32)[None, :]
    codes, scales = O.quantize_f32(x, gs)
    assert scales[0, 0] == 0x40                       # 2.0 in E4M3
    assert np.array_equal(O.dequantize(codes, scales, gs), x)


def test_bf16_entry_matches_f32_entry():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, (16, 64)).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    xb = bf16_bits_to_f32(bits)
    gs = O.global_scale_bf16(bits)
    c1, s1 = O.quantize_bf16(bits, gs)
    c2, s2 = O.quantize_f32(xb, gs)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    assert gs == O.global_scale_from_amax(np.abs(xb).max())


@pytest.mark.parametrize("cols", [16, 48, 256])
def test_dequantize_exact_product(cols):
    rng = np.random.default_rng(cols)
    codes = rng.integers(0, 256, (3, cols // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, (3, cols // 16), dtype=np.uint8)
    gs = np.float32(3.0)
    dq = O.dequantize(codes, scales, gs)
    want = (E2M1_VALUE[unpack_codes(codes)] * np.repeat(e4m3_value(scales), 16, axis=1)).astype(np.float32) / gs
    assert np.array_equal(dq, want.astype(np.float32))
