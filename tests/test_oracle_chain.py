"""Pins for the oracle's routing, GEMM and MoE chain (CPU only).

Routing is checked against numpy's stable argsort and bincount; the GEMM
against numpy's matmul on the dequantised operands; the MoE chain against a
brute-force per-token loop (each token runs its k experts as dense MLPs) built
from library primitives, and against its one-expert dense reduction.
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_moe_expert_topk_b200 import workloads as W


def test_route_matches_stable_sort():
    rng = np.random.default_rng(0)
    for E, R in [(8, 128), (48, 384), (384, 24576), (5, 3)]:
        ids = rng.integers(0, E, R).astype(np.int32)
        r = O.route(ids, E)
        assert np.array_equal(r["counts"], np.bincount(ids, minlength=E))
        assert r["offsets"][0] == 0 and np.array_equal(np.diff(r["offsets"]), r["counts"])
        order = np.argsort(ids, kind="stable")             # library stable sort
        pos = np.empty(R, np.int64)
        pos[order] = np.arange(R)
        assert np.array_equal(r["offsets"][ids] + r["rank"], pos)
        pad = ((r["counts"] + 127) // 128) * 128
        assert np.array_equal(np.diff(r["padded_offsets"]), pad)
        assert np.array_equal(r["pos_padded"], r["padded_offsets"][ids] + r["rank"])
        assert r["bad"] == 0


def test_route_skips_negative_and_flags_out_of_range():
    ids = np.array([2, -1, 0, 7, 2, 3, -5, 2], np.int32)
    r = O.route(ids, 4)
    assert r["bad"] == 1
    assert r["counts"].tolist() == [1, 0, 3, 1]
    assert r["rank"].tolist() == [0, -1, 0, -1, 1, 0, -1, 2]
    assert r["pos_padded"].tolist() == [128, -1, 0, -1, 129, 256, -1, 130]


def _quantize_bf16_tensor(t, gs=None):
    bits = W.bf16_bits(t)
    if gs is None:
        gs = O.global_scale_bf16(bits)
    c, s = O.quantize_bf16(bits, gs)
    return c, s, np.float32(gs)


def test_gemm_matches_numpy_matmul_with_segments():
    g = torch.Generator().manual_seed(1)
    M, N, K = 40, 96, 128
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b[64:] *= 30                                          # second segment on another scale
    ac, as_, ag = _quantize_bf16_tensor(a)
    b1c, b1s, b1g = _quantize_bf16_tensor(b[:64])
    b2c, b2s, b2g = _quantize_bf16_tensor(b[64:])
    bc, bs = np.concatenate([b1c, b2c]), np.concatenate([b1s, b2s])
    out = O.gemm(ac, as_, ag, bc, bs, [b1g, b2g], [64, 96])
    A = O.dequantize(ac, as_, ag).astype(np.float64)
    B = np.concatenate([O.dequantize(b1c, b1s, b1g), O.dequantize(b2c, b2s, b2g)]).astype(np.float64)
    ref = np.matmul(A, B.T)
    assert np.allclose(out, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())
    # a transposed operand or swapped segment scale would not match:
    assert not np.allclose(out[:, 64:], np.matmul(A, B.T)[:, 64:] * (b1g / b2g), rtol=1e-3)


def test_gemm_one_hot_probe_is_exact():
    K = 64
    a_codes = np.zeros((1, K // 2), np.uint8)
    a_codes[0, 5] = 0x30                       # element 11 = code 3 (1.5)
    a_scales = np.full((1, K // 16), 0x38, np.uint8)   # 1.0
    b_codes = np.zeros((2, K // 2), np.uint8)
    b_codes[1, 5] = 0x70                       # element 11 of row 1 = 6.0
    b_scales = np.full((2, K // 16), 0x40, np.uint8)   # 2.0
    out = O.gemm(a_codes, a_scales, 2.0, b_codes, b_scales, [4.0])
    assert out.tolist() == [[0.0, 1.5 * 1.0 / 2.0 * 6.0 * 2.0 / 4.0]]


def _tiny_problem(E=4, k=2, T=12, H=64, I=32, seed=0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(T, H, generator=g)).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g)
    w, ids = torch.topk(torch.softmax(logits, -1), k, dim=-1)
    ids = ids.to(torch.int32)
    w = (w / w.sum(-1, keepdim=True)).float()
    w13 = (torch.randn(E, 2 * I, H, generator=g) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g) * 0.02).to(torch.bfloat16)
    xc, xs, xg = _quantize_bf16_tensor(x)
    w13c, w13s, w13g, w2c, w2s, w2g = [], [], [], [], [], []
    for e in range(E):
        gc, gsc, gg = _quantize_bf16_tensor(w13[e, :I])
        uc, usc, ug = _quantize_bf16_tensor(w13[e, I:])
        dc, dsc, dg = _quantize_bf16_tensor(w2[e])
        w13c.append(np.concatenate([gc, uc])); w13s.append(np.concatenate([gsc, usc]))
        w13g.append([gg, ug]); w2c.append(dc); w2s.append(dsc); w2g.append(dg)
    P = dict(x_bits=W.bf16_bits(x), topk_ids=ids.numpy(), topk_weights=w.numpy(), x_gs=xg,
             w13_codes=np.stack(w13c), w13_scales=np.stack(w13s), w13_gs=np.array(w13g, np.float32),
             w2_codes=np.stack(w2c), w2_scales=np.stack(w2s), w2_gs=np.array(w2g, np.float32))
    return P, (E, k, T, H, I)


def _brute_force(P, inter_gs, dims, x_codes=None, x_scales=None):
    """Per token, per slot: dense expert MLP on dequantised operands (numpy
    matmul, torch SiLU), re-quantised with the oracle's pinned quantiser.
    With x_codes / x_scales, those stand for the quantised activations."""
    E, k, T, H, I = dims
    if x_codes is None:
        xc, xs = O.quantize_bf16(P["x_bits"], P["x_gs"])
    else:
        xc, xs = x_codes, x_scales
    A = O.dequantize(xc, xs, P["x_gs"]).astype(np.float64)
    out = np.zeros((T, H))
    h_amax = np.zeros(E, np.float32)
    hs = {}
    for t in range(T):
        for j in range(k):
            e = int(P["topk_ids"][t, j])
            Wg = O.dequantize(P["w13_codes"][e][:I], P["w13_scales"][e][:I], P["w13_gs"][e][0]).astype(np.float64)
            Wu = O.dequantize(P["w13_codes"][e][I:], P["w13_scales"][e][I:], P["w13_gs"][e][1]).astype(np.float64)
            g = np.matmul(Wg, A[t]).astype(np.float32)
            u = np.matmul(Wu, A[t]).astype(np.float32)
            h = (torch.nn.functional.silu(torch.from_numpy(g).double()) * torch.from_numpy(u).double()).float().numpy()
            hs[(t, j)] = h
            h_amax[e] = max(h_amax[e], np.abs(h).max())
            if inter_gs is None:
                continue
            hc, hsc = O.quantize_f32(h[None, :], inter_gs[e])
            hd = O.dequantize(hc, hsc, inter_gs[e]).astype(np.float64)[0]
            W2 = O.dequantize(P["w2_codes"][e], P["w2_scales"][e], P["w2_gs"][e]).astype(np.float64)
            y = np.matmul(W2, hd).astype(np.float32)
            out[t] += float(P["topk_weights"][t, j]) * y
    return out, h_amax, hs


def test_moe_forward_equals_per_token_brute_force():
    P, dims = _tiny_problem()
    E = dims[0]
    inter_gs = O.moe_warmup_inter_gs(**P)
    out, inter = O.moe_forward(**P, inter_gs=inter_gs, intermediates=True)
    ref, h_amax, hs = _brute_force(P, inter_gs, dims)
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    assert np.array_equal(inter["h_amax"], h_amax)
    want_gs = np.array([O.global_scale_from_amax(a) for a in h_amax], np.float32)
    assert np.array_equal(inter_gs, want_gs)
    k = dims[1]
    for (t, j), h in hs.items():
        assert np.array_equal(inter["h"][t * k + j], h)


def test_moe_forward_gate_up_order_matters():
    """Swapping gate and up halves changes the result (the pin above would
    catch an oracle that used them the other way round)."""
    P, dims = _tiny_problem(seed=3)
    E, k, T, H, I = dims
    inter_gs = O.moe_warmup_inter_gs(**P)
    out = O.moe_forward(**P, inter_gs=inter_gs)
    Q = dict(P)
    Q["w13_codes"] = np.concatenate([P["w13_codes"][:, I:], P["w13_codes"][:, :I]], axis=1)
    Q["w13_scales"] = np.concatenate([P["w13_scales"][:, I:], P["w13_scales"][:, :I]], axis=1)
    Q["w13_gs"] = P["w13_gs"][:, ::-1].copy()
    out2 = O.moe_forward(**Q, inter_gs=inter_gs)
    assert np.abs(out - out2).max() > 1e-3 * np.abs(out).max()


def test_moe_single_expert_reduces_to_dense_chain():
    P, dims = _tiny_problem(E=1, k=1, T=9, H=64, I=32, seed=5)
    P["topk_weights"] = np.ones_like(P["topk_weights"])
    E, k, T, H, I = dims
    inter_gs = O.moe_warmup_inter_gs(**P)
    out = O.moe_forward(**P, inter_gs=inter_gs)
    xc, xs = O.quantize_bf16(P["x_bits"], P["x_gs"])
    G = O.gemm(xc, xs, P["x_gs"], P["w13_codes"][0], P["w13_scales"][0], P["w13_gs"][0], [I, 2 * I])
    g, u = G[:, :I], G[:, I:]
    h = (torch.nn.functional.silu(torch.from_numpy(g).double()) * torch.from_numpy(u).double()).float().numpy()
    hc, hs = O.quantize_f32(h, inter_gs[0])
    y = O.gemm(hc, hs, inter_gs[0], P["w2_codes"][0], P["w2_scales"][0], P["w2_gs"][0:1])
    np.testing.assert_allclose(out, y, rtol=1e-6, atol=1e-7 * np.abs(y).max())


def test_shared_expert_folded_equals_routed_plus_dense_chain():
    """The shared expert folded in as one more group (reading R13: slot k is
    expert E with weight 1, ids from the oracle router) gives the routed
    chain's output plus the shared expert's dense chain (the one-expert
    reduction pinned above), up to the fp32 rounding of the two partial sums."""
    P, dims = _tiny_problem(E=5, k=2, T=10, seed=11)
    E, k, T, H, I = dims
    Er = E - 1                                            # routed experts 0..3, shared expert 4
    logits = np.random.default_rng(4).normal(0, 1, (T, Er)).astype(np.float32)
    ids, w = O.topk(logits, k, "softmax", num_shared=1)
    assert (ids[:, :k] < Er).all() and (ids[:, k] == Er).all()
    folded = dict(P, topk_ids=ids, topk_weights=w)
    inter_gs = O.moe_warmup_inter_gs(**folded)
    out = O.moe_forward(**folded, inter_gs=inter_gs)
    routed = O.moe_forward(**dict(P, topk_ids=ids[:, :k].copy(), topk_weights=w[:, :k].copy()), inter_gs=inter_gs)
    shared = O.moe_forward(**dict(P, topk_ids=ids[:, k:].copy(), topk_weights=w[:, k:].copy()), inter_gs=inter_gs)
    np.testing.assert_allclose(out, routed.astype(np.float64) + shared, rtol=1e-6,
                               atol=1e-7 * np.abs(out).max())
    # the shared part is the dense chain of expert 4 on every token
    xc, xs = O.quantize_bf16(P["x_bits"], P["x_gs"])
    G = O.gemm(xc, xs, P["x_gs"], P["w13_codes"][Er], P["w13_scales"][Er], P["w13_gs"][Er], [I, 2 * I])
    g, u = G[:, :I], G[:, I:]
    h = (torch.nn.functional.silu(torch.from_numpy(g).double()) * torch.from_numpy(u).double()).float().numpy()
    hc, hs = O.quantize_f32(h, inter_gs[Er])
    y = O.gemm(hc, hs, inter_gs[Er], P["w2_codes"][Er], P["w2_scales"][Er], P["w2_gs"][Er:Er + 1])
    np.testing.assert_allclose(shared, y, rtol=1e-6, atol=1e-7 * np.abs(y).max())
    # and the shared expert's contribution is not negligible
    assert np.abs(shared).max() > 0.1 * np.abs(routed).max()


def test_moe_skipped_slots_contribute_nothing():
    P, dims = _tiny_problem(seed=7)
    inter_gs = O.moe_warmup_inter_gs(**P)
    full = O.moe_forward(**P, inter_gs=inter_gs)
    Q = dict(P)
    ids = P["topk_ids"].copy()
    ids[:, 1] = -1
    Q["topk_ids"] = ids
    part = O.moe_forward(**Q, inter_gs=inter_gs)
    Q["topk_ids"] = P["topk_ids"][:, :1].copy()
    Q["topk_weights"] = P["topk_weights"][:, :1].copy()
    one = O.moe_forward(**Q, inter_gs=inter_gs)
    np.testing.assert_array_equal(part, one)
    assert np.abs(full - part).max() > 0


def test_warmup_fallback_for_experts_without_rows():
    P, dims = _tiny_problem(E=4, k=1, T=6, seed=2)
    P["topk_ids"] = np.array([[0], [0], [2], [2], [0], [2]], np.int32)
    P["topk_weights"] = np.ones((6, 1), np.float32)
    inter_gs = O.moe_warmup_inter_gs(**P)
    _, inter = O.moe_forward(**P, inter_gs=inter_gs, intermediates=True)
    amax = inter["h_amax"]
    assert amax[1] == 0 and amax[3] == 0
    assert inter_gs[1] == inter_gs[3] == O.global_scale_from_amax(max(amax[0], amax[2]))


def test_moe_forward_on_given_codes_equals_brute_force():
    """Activations given already in NVFP4 (expert-parallel dispatch of 4-bit
    rows): arbitrary codes and scales, not those of any bf16 x, go through
    the same chain as the brute force built from them; with the codes of x
    itself the output is the bf16 path's bit for bit."""
    P, dims = _tiny_problem(seed=3)
    E, k, T, H, I = dims
    rng = np.random.default_rng(3)
    xc = rng.integers(0, 256, (T, H // 2), dtype=np.uint8)
    xs = rng.integers(0x28, 0x48, (T, H // 16), dtype=np.uint8)      # E4M3 scales 0.25 .. 4
    Q = dict(P, x_gs=np.float32(3.0))
    _, h_amax, _ = _brute_force(Q, None, dims, xc, xs)
    inter_gs = np.array([O.global_scale_from_amax(a if a > 0 else h_amax.max()) for a in h_amax], np.float32)
    out = O.moe_forward(**Q, inter_gs=inter_gs, x_codes=xc, x_scales=xs)
    ref, _, _ = _brute_force(Q, inter_gs, dims, xc, xs)
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    own_c, own_s = O.quantize_bf16(P["x_bits"], P["x_gs"])
    inter_gs = O.moe_warmup_inter_gs(**P)
    assert np.array_equal(O.moe_forward(**P, inter_gs=inter_gs, x_codes=own_c, x_scales=own_s),
                          O.moe_forward(**P, inter_gs=inter_gs))
