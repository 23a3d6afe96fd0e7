"""GPU parity of the integer / byte steps: global scale, quantisation, scale
layout, routing.  All bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import from_mma_layout, to_mma_layout
from nvfp4_moe_expert_topk_b200 import (NVFP4_SCALES_MMA, NVFP4_SCALES_ROWMAJOR, nvfp4_global_scale,
                                        nvfp4_moe_get_error, nvfp4_moe_route_debug, nvfp4_quantize,
                                        nvfp4_scales_bytes, nvfp4_swizzle_scales)
from nvfp4_moe_expert_topk_b200 import prep
from nvfp4_moe_expert_topk_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def special_matrix(rows, cols, seed):
    """bf16 values with per-row magnitude spread, zero blocks, tiny blocks,
    exact E2M1 ties and negative zeros."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * torch.exp(torch.empty(rows, 1).uniform_(-8, 8, generator=g))
    if cols >= 32:
        x[0, :16] = 0.0
        x[min(1, rows - 1), 16:32] = 1e-30
    if rows > 2 and cols >= 16:
        x[2, :16] = torch.tensor([3.0, 0.3, -0.375, 1.25, 0.0, -3.0, 0.1, -0.1, 1.0, 0.875, 2.0, -2.5,
                                  0.625, 1.5, -1.5, 0.75])
    if rows > 3 and cols >= 16:
        x[3, :16] = -0.0
        x[3, 0] = -1.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("shape,seed", [((1, 16), 0), ((3, 48), 1), ((37, 256), 2), ((300, 7168), 3),
                                        ((8, 1000 * 16), 4)])
def test_global_scale_bitexact(shape, seed):
    x = special_matrix(*shape, seed)
    gs = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(x.to(DEV), gs)
    assert gs.item() == O.global_scale_bf16(W.bf16_bits(x))
    # odd length, unaligned start
    flat = x.reshape(-1).to(DEV)
    sub = flat[1:flat.numel() - 2]
    nvfp4_global_scale(sub, gs)
    assert gs.item() == O.global_scale_bf16(W.bf16_bits(x).reshape(-1)[1:-2])
    nvfp4_global_scale(torch.zeros(17, dtype=torch.bfloat16, device=DEV), gs)
    assert gs.item() == 1.0


@pytest.mark.parametrize("shape,seed", [((1, 16), 0), ((3, 48), 1), ((37, 256), 2), ((300, 7168), 3),
                                        ((129, 3072), 5)])
def test_quantize_rowmajor_bitexact(shape, seed):
    rows, cols = shape
    x = special_matrix(rows, cols, seed)
    bits = W.bf16_bits(x)
    gs = O.global_scale_bf16(bits)
    want_c, want_s = O.quantize_bf16(bits, gs)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=DEV)
    nvfp4_quantize(x.to(DEV), torch.tensor([gs], device=DEV), codes, scales, NVFP4_SCALES_ROWMAJOR)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)


@pytest.mark.parametrize("rows,cols", [(1, 64), (130, 256), (300, 7168)])
def test_quantize_mma_layout_bitexact(rows, cols):
    x = special_matrix(rows, cols, rows)
    bits = W.bf16_bits(x)
    gs = O.global_scale_bf16(bits)
    want_c, want_s = O.quantize_bf16(bits, gs)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(nvfp4_scales_bytes(rows, cols, NVFP4_SCALES_MMA), dtype=torch.uint8, device=DEV)
    nvfp4_quantize(x.to(DEV), torch.tensor([gs], device=DEV), codes, scales, NVFP4_SCALES_MMA)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    buf = scales.cpu().numpy()
    np.testing.assert_array_equal(from_mma_layout(buf, rows, cols), want_s)
    np.testing.assert_array_equal(buf, to_mma_layout(want_s))      # pad rows untouched (zero)


def test_quantize_oversized_global_scale():
    """The pages' NaN case: multiplier 3977.6 on activations of amax ~1.27
    ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 2, "What the quant method
    does"): saturating conversion gives 448 scales and finite codes."""
    g = torch.Generator().manual_seed(0)
    x = (torch.rand(64, 256, generator=g) * 2.54 - 1.27).to(torch.bfloat16)
    bits = W.bf16_bits(x)
    gs = np.float32(3977.6)
    want_c, want_s = O.quantize_bf16(bits, gs)
    codes = torch.empty(64, 128, dtype=torch.uint8, device=DEV)
    scales = torch.empty(64, 16, dtype=torch.uint8, device=DEV)
    nvfp4_quantize(x.to(DEV), torch.tensor([gs], device=DEV), codes, scales, NVFP4_SCALES_ROWMAJOR)
    s = scales.cpu().numpy()
    np.testing.assert_array_equal(s, want_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    assert (s == 0x7E).mean() > 0.9 and not np.any((s & 0x7F) == 0x7F)


def test_swizzle_kernel_matches_layout_definition():
    g = np.random.default_rng(0)
    for batch, rows, cols in [(1, 128, 64), (3, 200, 256), (2, 6144, 7168)]:
        sc = g.integers(0, 0x7F, (batch, rows, cols // 16), dtype=np.uint8)
        out = torch.full((batch * nvfp4_scales_bytes(rows, cols, NVFP4_SCALES_MMA),), 0xAA, dtype=torch.uint8,
                         device=DEV)
        nvfp4_swizzle_scales(torch.from_numpy(sc).to(DEV), out, batch, rows, cols)
        got = out.cpu().numpy().reshape(batch, -1)
        for b in range(batch):
            np.testing.assert_array_equal(got[b], to_mma_layout(sc[b]))


@pytest.mark.parametrize("E,T,k,seed", [(8, 64, 2, 0), (48, 64, 6, 1), (384, 4096, 6, 2), (5, 3, 2, 3),
                                        (1, 256, 1, 4), (1024, 300, 8, 5), (64, 20011, 8, 6), (3, 1, 3, 7),
                                        (1024, 4099, 32, 8)])
def test_route_bitexact(E, T, k, seed):
    """Routing (one launch over min(T, SMs) blocks, each owning a contiguous
    token range) against the oracle's stable counting sort: one token; T not
    a multiple of the block count; ~1000 slots per block; 1024 experts."""
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    if E == 384:                                  # skewed, with empty experts
        cfg = W.MOE_CONFIGS["prefill"]
        ids = W.routing(cfg)[0].numpy()
    ref = O.route(ids, E)
    ws = prep.workspace(T, k, E, 128, 128, DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    poff = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    nvfp4_moe_route_debug(torch.from_numpy(ids).to(DEV), E, counts, poff, inv, ws)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(poff.cpu().numpy(), ref["padded_offsets"])
    np.testing.assert_array_equal(inv.cpu().numpy(), ref["pos_padded"])
    assert nvfp4_moe_get_error(ws) == 0


def test_route_skipped_and_bad_ids():
    ids = np.array([[2, -1], [0, 7], [2, 3], [-5, 2]], np.int32)
    E = 4
    ref = O.route(ids, E)
    ws = prep.workspace(4, 2, E, 128, 128, DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    poff = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    inv = torch.empty(8, dtype=torch.int32, device=DEV)
    nvfp4_moe_route_debug(torch.from_numpy(ids).to(DEV), E, counts, poff, inv, ws)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(inv.cpu().numpy(), ref["pos_padded"])
    assert nvfp4_moe_get_error(ws) == -8          # NVFP4_ERR_BAD_EXPERT_ID, sticky until read
    assert nvfp4_moe_get_error(ws) == 0           # read clears it


@pytest.mark.parametrize("seed", range(24))
def test_route_random_shapes(seed):
    """Seeded random E (1-1024), k (1-min(32, E)), T (1-5000) with about a
    tenth of the slots skipped (-1) and, every fourth seed, Zipf-like skew:
    counts, padded offsets and every slot's padded row bit-exact."""
    rng = np.random.default_rng(5000 + seed)
    E = int(rng.integers(1, 1025))
    k = int(rng.integers(1, min(32, E) + 1))
    T = int(rng.integers(1, 5001))
    if seed % 4 == 0:
        p = 1.0 / np.arange(1, E + 1) ** 1.2
        ids = rng.choice(E, size=(T, k), p=p / p.sum()).astype(np.int32)
    else:
        ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[rng.random((T, k)) < 0.1] = -1
    ref = O.route(ids, E)
    ws = prep.workspace(T, k, E, 128, 128, DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    poff = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    nvfp4_moe_route_debug(torch.from_numpy(ids).to(DEV), E, counts, poff, inv, ws)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(poff.cpu().numpy(), ref["padded_offsets"])
    np.testing.assert_array_equal(inv.cpu().numpy(), ref["pos_padded"])
    assert nvfp4_moe_get_error(ws) == 0


@pytest.mark.parametrize("seed", range(16))
def test_quantize_random_shapes(seed):
    """Seeded random rows (1-700) and columns (a multiple of 64 up to 8192) of
    special values, both scale layouts: codes and scales bit-exact."""
    rng = np.random.default_rng(6000 + seed)
    rows = int(rng.integers(1, 701))
    cols = 64 * int(rng.integers(1, 129))
    x = special_matrix(rows, cols, 7000 + seed)
    bits = W.bf16_bits(x)
    gs = O.global_scale_bf16(bits)
    want_c, want_s = O.quantize_bf16(bits, gs)
    xd, g = x.to(DEV), torch.tensor([gs], device=DEV)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=DEV)
    nvfp4_quantize(xd, g, codes, scales, NVFP4_SCALES_ROWMAJOR)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    mma = torch.zeros(nvfp4_scales_bytes(rows, cols, NVFP4_SCALES_MMA), dtype=torch.uint8, device=DEV)
    nvfp4_quantize(xd, g, codes, mma, NVFP4_SCALES_MMA)
    np.testing.assert_array_equal(from_mma_layout(mma.cpu().numpy(), rows, cols), want_s)


@pytest.mark.parametrize("rows,cols,ldx", [(37, 256, 264), (130, 1024, 1536), (5, 64, 72)])
def test_quantize_strided_rows(rows, cols, ldx):
    """The C ABI's ldx > cols: x is a [rows, cols] window of a wider bf16
    buffer (the columns past cols hold huge values that must not enter any
    block's amax); codes and scales equal the contiguous window's, bit for bit."""
    import ctypes
    from nvfp4_moe_expert_topk_b200 import lib
    x = special_matrix(rows, cols, rows + cols)
    bits = W.bf16_bits(x)
    gs = O.global_scale_bf16(bits)
    want_c, want_s = O.quantize_bf16(bits, gs)
    wide = torch.full((rows, ldx), 30000.0, dtype=torch.bfloat16)
    wide[:, :cols] = x
    wd = wide.to(DEV)
    g = torch.tensor([gs], device=DEV)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=DEV)
    P = ctypes.c_void_p
    st = lib().nvfp4_quantize(P(wd.data_ptr()), rows, cols, ldx, P(g.data_ptr()), P(codes.data_ptr()),
                              P(scales.data_ptr()), NVFP4_SCALES_ROWMAJOR,
                              P(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == 0
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
