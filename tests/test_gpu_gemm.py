"""GPU parity of the dense NVFP4 GEMM (the grouped engine with one group):
one-hot probes that pin nibble order, scale placement and the B halves, then
random problems against the oracle, including ragged M, a partial last
k-tile and dual global scales."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import bf16_to_np, cosine, row_rel_l2, to_mma_layout
from nvfp4_moe_expert_topk_b200 import nvfp4_gemm
from nvfp4_moe_expert_topk_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"

E2M1 = [0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6]


def run_gemm(a_codes, a_sc, a_gs, b_codes, b_sc, b_gs, seg_end):
    M, N = a_codes.shape[0], b_codes.shape[0]
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    nvfp4_gemm(torch.from_numpy(a_codes).to(DEV), torch.from_numpy(to_mma_layout(a_sc)).to(DEV),
               torch.tensor([a_gs], dtype=torch.float32, device=DEV), torch.from_numpy(b_codes).to(DEV),
               torch.from_numpy(to_mma_layout(b_sc)).to(DEV),
               torch.tensor(np.asarray(b_gs, np.float32), device=DEV), seg_end, out)
    torch.cuda.synchronize()
    return bf16_to_np(out)


def set_code(codes, r, k, c):
    b = codes[r, k // 2]
    codes[r, k // 2] = (b & 0xF0) | c if k % 2 == 0 else (b & 0x0F) | (c << 4)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (128, 128, 512), (200, 512, 1024)])
def test_one_hot_probes(M, N, K):
    rng = np.random.default_rng(M + N + K)
    for trial in range(6):
        m0, n0, k0 = int(rng.integers(M)), int(rng.integers(N)), int(rng.integers(K))
        ca, cb = int(rng.integers(1, 16)), int(rng.integers(1, 16))
        a = np.zeros((M, K // 2), np.uint8)
        b = np.zeros((N, K // 2), np.uint8)
        set_code(a, m0, k0, ca)
        set_code(b, n0, k0, cb)
        a_sc = np.full((M, K // 16), 0x38, np.uint8)        # 1.0
        b_sc = np.full((N, K // 16), 0x38, np.uint8)
        sa, sb = [0x30, 0x40, 0x48][trial % 3], [0x38, 0x44, 0x2C][trial % 3]   # 0.5/2/4, 1/3/0.1875
        a_sc[m0, k0 // 16] = sa
        b_sc[n0, k0 // 16] = sb
        out = run_gemm(a, a_sc, 1.0, b, b_sc, [2.0], [N])
        want = np.zeros((M, N), np.float32)
        want[m0, n0] = E2M1[ca] * O.e4m3_decode(sa) * E2M1[cb] * O.e4m3_decode(sb) / 2.0
        np.testing.assert_array_equal(out, want.astype(np.float32))


def quantized_operands(M, N, K, seed, segs):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = torch.randn(N, K, generator=g) * 0.02
    start = 0
    for i, end in enumerate(segs):
        b[start:end] *= (1.0, 30.0, 0.1, 3.0)[i]
        start = end
    b = b.to(torch.bfloat16)
    ab = W.bf16_bits(a)
    a_gs = O.global_scale_bf16(ab)
    ac, asc = O.quantize_bf16(ab, a_gs)
    bc, bsc, bgs = [], [], []
    start = 0
    for end in segs:
        part = W.bf16_bits(b[start:end])
        gs = O.global_scale_bf16(part)
        c, s = O.quantize_bf16(part, gs)
        bc.append(c), bsc.append(s), bgs.append(gs)
        start = end
    return ac, asc, a_gs, np.concatenate(bc), np.concatenate(bsc), np.array(bgs, np.float32)


@pytest.mark.parametrize("M,N,K,segs", [
    (128, 256, 256, [256]),
    (1, 128, 64, [128]),            # single row, one k-block
    (64, 256, 192, [256]),          # partial last k-tile (3 of 4 k-blocks)
    (200, 384, 512, [128, 384]),    # ragged M, N % 256 != 0, two global scales
    (257, 512, 1536, [256, 512]),   # q_b-like K
    (130, 2048, 7168, [1536, 2048]),  # fused_wqa_wkv-like: dual global scales split at 1536
    (300, 1024, 8192, [1024]),      # o_b-like K
])
def test_gemm_matches_oracle(M, N, K, segs):
    ac, asc, a_gs, bc, bsc, bgs = quantized_operands(M, N, K, M * 7 + N, segs)
    ref = O.gemm(ac, asc, a_gs, bc, bsc, bgs, segs)
    out = run_gemm(ac, asc, a_gs, bc, bsc, bgs, segs)
    assert np.all(np.isfinite(out))
    err = row_rel_l2(out, ref)
    assert err.max() <= 5e-3, err.max()
    assert cosine(out, ref) >= 0.99999


@pytest.mark.parametrize("name", ["wqa_wkv", "q_b", "o_b"])
def test_mla_projection_full_size(name):
    """The MLA projections at M=2048 ("nvfp4-megamoe-kernel / CURRENT_BUG.md",
    page 1 "Phase 2", option 1: one NVFP4 GEMM per projection; fused_wqa_wkv
    with one global scale per half).  The device quantises activation and
    weight through the library; both equal the oracle's quantisation bit for
    bit; sampled output rows match the oracle GEMM."""
    from nvfp4_moe_expert_topk_b200 import NVFP4_SCALES_MMA, nvfp4_global_scale, nvfp4_quantize, nvfp4_scales_bytes
    from helpers import from_mma_layout
    idx = list(W.MLA_GEMMS).index(name)
    cfg = W.MLA_GEMMS[name]
    a, w = W.gemm_operands(cfg, idx, DEV)
    M, N, K = cfg.M, cfg.N, cfg.K
    # device quantisation (activation: one global scale; weight: one per segment)
    ad = a.to(DEV)
    a_gs = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(ad, a_gs)
    a_codes = torch.empty(M, K // 2, dtype=torch.uint8, device=DEV)
    a_sc = torch.empty(nvfp4_scales_bytes(M, K, NVFP4_SCALES_MMA), dtype=torch.uint8, device=DEV)
    nvfp4_quantize(ad, a_gs, a_codes, a_sc, NVFP4_SCALES_MMA)
    w_codes = torch.empty(N, K // 2, dtype=torch.uint8, device=DEV)
    w_sc = torch.empty(nvfp4_scales_bytes(N, K, NVFP4_SCALES_MMA), dtype=torch.uint8, device=DEV)
    segs = list(cfg.seg_end)
    w_gs = torch.empty(len(segs), dtype=torch.float32, device=DEV)
    start = 0
    for i, end in enumerate(segs):
        nvfp4_global_scale(w[start:end], w_gs[i:i + 1])
        nvfp4_quantize(w[start:end], w_gs[i:i + 1], w_codes[start:end],
                       w_sc[start * (K // 16):end * (K // 16)], NVFP4_SCALES_MMA)
        start = end
    out = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nvfp4_gemm(a_codes, a_sc, a_gs, w_codes, w_sc, w_gs, segs, out)
    torch.cuda.synchronize()
    # oracle quantisation of the same bf16 values
    ab = W.bf16_bits(a)
    oa_gs = O.global_scale_bf16(ab)
    assert a_gs.item() == oa_gs
    oac, oas = O.quantize_bf16(ab, oa_gs)
    np.testing.assert_array_equal(a_codes.cpu().numpy(), oac)
    np.testing.assert_array_equal(from_mma_layout(a_sc.cpu().numpy(), M, K), oas)
    wb = W.bf16_bits(w)
    owc, ows, owg = [], [], []
    start = 0
    for i, end in enumerate(segs):
        gs = O.global_scale_bf16(wb[start:end])
        assert w_gs[i].item() == gs
        c, s_ = O.quantize_bf16(wb[start:end], gs)
        owc.append(c), ows.append(s_), owg.append(gs)
        start = end
    owc, ows = np.concatenate(owc), np.concatenate(ows)
    np.testing.assert_array_equal(w_codes.cpu().numpy(), owc)
    # sampled rows: first, last, and random ones across the m-tiles
    rows = np.unique(np.concatenate([[0, M - 1, 127, 128], np.random.default_rng(idx).choice(M, 4, replace=False)]))
    ref = O.gemm(oac[rows], oas[rows], oa_gs, owc, ows, np.array(owg, np.float32), segs)
    got = bf16_to_np(out[torch.from_numpy(rows).to(DEV)])
    err = row_rel_l2(got, ref)
    assert err.max() <= 5e-3, err.max()
    assert cosine(got, ref) >= 0.99999


@pytest.mark.parametrize("M,N,K,segs", [
    (256, 20480, 1024, [20480]),            # 80 pair tiles over 74 SM pairs: a second, nearly empty round
    (300, 10240, 512, [4096, 10240]),       # ragged M (empty half in each last pair), dual global scales
    (128, 40960, 512, [40960]),             # one m-tile: 160 one-CTA tiles over 148 SMs
    (2048, 7168, 8192, [7168]),             # o_b shape: 224 pair tiles over 74 pairs
])
def test_gemm_wide_shapes_match_oracle(M, N, K, segs):
    """Shapes whose tiles fill the GPU unevenly: sampled rows against the
    oracle, and two calls bit-identical (each element is one fp32 sum in a
    fixed k order)."""
    ac, asc, a_gs, bc, bsc, bgs = quantized_operands(M, N, K, M + N + K, segs)
    dev_args = (torch.from_numpy(ac).to(DEV), torch.from_numpy(to_mma_layout(asc)).to(DEV),
                torch.tensor([a_gs], dtype=torch.float32, device=DEV), torch.from_numpy(bc).to(DEV),
                torch.from_numpy(to_mma_layout(bsc)).to(DEV), torch.tensor(np.asarray(bgs, np.float32), device=DEV))
    outs = []
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        nvfp4_gemm(*dev_args, segs, out)
        torch.cuda.synchronize()
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    got = bf16_to_np(outs[0])
    assert np.all(np.isfinite(got))
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M).choice(M, 6, replace=False)]))
    ref = O.gemm(ac[rows], asc[rows], a_gs, bc, bsc, bgs, segs)
    err = row_rel_l2(got[rows], ref)
    assert err.max() <= 5e-3, err.max()


@pytest.mark.parametrize("M,N,K,segs", [
    (257, 512, 256, [512]),      # pair tiles (staged stores): ragged last pair, 1 row in its odd half
    (100, 384, 256, [384]),      # one-CTA tiles (direct stores)
])
def test_gemm_strided_output_leaves_the_rest(M, N, K, segs):
    """The C ABI's ldo > N: out is a window [M, N] of a wider buffer.  The
    window equals the contiguous call's result bit for bit; the columns past
    N and the row past M keep their sentinel."""
    import ctypes
    from nvfp4_moe_expert_topk_b200 import lib
    ac, asc, a_gs, bc, bsc, bgs = quantized_operands(M, N, K, M * 3 + N, segs)
    d = [torch.from_numpy(ac).to(DEV), torch.from_numpy(to_mma_layout(asc)).to(DEV),
         torch.tensor([a_gs], dtype=torch.float32, device=DEV), torch.from_numpy(bc).to(DEV),
         torch.from_numpy(to_mma_layout(bsc)).to(DEV), torch.tensor(np.asarray(bgs, np.float32), device=DEV)]
    plain = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nvfp4_gemm(*d, segs, plain)
    ldo = N + 72
    buf = torch.full((M + 1, ldo), 7.0, dtype=torch.bfloat16, device=DEV)
    seg = (ctypes.c_int64 * len(segs))(*segs)
    st = lib().nvfp4_gemm(*[ctypes.c_void_p(t.data_ptr()) for t in d[:3]], M,
                          *[ctypes.c_void_p(t.data_ptr()) for t in d[3:]], ctypes.cast(seg, ctypes.c_void_p), len(segs),
                          N, K, ctypes.c_void_p(buf.data_ptr()), ldo,
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == 0
    assert torch.equal(buf[:M, :N], plain)
    assert bool((buf[:M, N:] == 7.0).all())
    assert bool((buf[M] == 7.0).all())


@pytest.mark.parametrize("seed", range(24))
def test_random_dense_shapes_match_oracle(seed):
    """Dense GEMMs of seeded random shapes (M 1-700, N a multiple of 128 up to
    1024, K a multiple of 64 up to 1024, 1-3 global-scale segments): every
    output row against the oracle, on whichever tiles the plan picks (pairs
    with staged TMA stores when M > 128 and N % 256 == 0)."""
    rng = np.random.default_rng(2000 + seed)
    M = int(rng.integers(1, 701))
    N = 128 * int(rng.integers(1, 9))
    K = 64 * int(rng.integers(1, 17))
    nseg = int(rng.integers(1, 4))
    cuts = sorted(set(int(c) for c in rng.integers(1, N // 32, size=nseg - 1) * 32)) if N >= 64 else []
    segs = [c for c in cuts if 0 < c < N] + [N]
    ac, asc, a_gs, bc, bsc, bgs = quantized_operands(M, N, K, 3000 + seed, segs)
    ref = O.gemm(ac, asc, a_gs, bc, bsc, bgs, segs)
    out = run_gemm(ac, asc, a_gs, bc, bsc, bgs, segs)
    assert np.all(np.isfinite(out))
    assert row_rel_l2(out, ref).max() <= 5e-3
    assert cosine(out, ref) >= 0.99999


def test_gemm_in_cuda_graph_with_new_inputs():
    """nvfp4_gemm (pair tiles with staged TMA stores: the output's tensor map
    is a launch parameter) captured once in a CUDA graph; replayed after new
    operands are copied into the captured buffers, it equals an eager call on
    those operands bit for bit."""
    M, N, K, segs = 300, 1024, 512, [512, 1024]
    first = quantized_operands(M, N, K, 11, segs)
    second = quantized_operands(M, N, K, 12, segs)

    def dev(ops):
        ac, asc, a_gs, bc, bsc, bgs = ops
        return [torch.from_numpy(ac).to(DEV), torch.from_numpy(to_mma_layout(asc)).to(DEV),
                torch.tensor([a_gs], dtype=torch.float32, device=DEV), torch.from_numpy(bc).to(DEV),
                torch.from_numpy(to_mma_layout(bsc)).to(DEV), torch.tensor(np.asarray(bgs, np.float32), device=DEV)]

    bufs = dev(first)
    out = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nvfp4_gemm(*bufs, segs, out)                      # eager call first (kernel attributes)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            nvfp4_gemm(*bufs, segs, out, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for b, n in zip(bufs, dev(second)):
        b.copy_(n)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    ref = torch.empty_like(out)
    nvfp4_gemm(*dev(second), segs, ref)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
