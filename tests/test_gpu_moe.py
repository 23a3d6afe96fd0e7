"""GPU parity of the whole routed-expert chain (nvfp4_moe_forward) against
the oracle on the same quantised operands.

Bars: routing, x codes and x scales bit-exact; output per row
||gpu - ref||_2 / ||ref||_2 <= 2e-2 and cosine >= 0.9995; h codes (which
depend on fp32 accumulation order) >= 99% identical with every mismatch an
adjacent code; the L2 GEMM fed the GPU's own h within 5e-3 per row."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import (OracleWeights, bf16_to_np, cosine, from_mma_layout, from_rowblock_layout, row_max_rel,
                     row_rel_l2)
from nvfp4_moe_expert_topk_b200 import (nvfp4_global_scale, nvfp4_moe_calibrate, nvfp4_moe_forward,
                                        nvfp4_moe_get_error, nvfp4_moe_workspace_region)
from nvfp4_moe_expert_topk_b200 import prep
from nvfp4_moe_expert_topk_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROW_TOL = 2e-2
COS_TOL = 0.9995


class Problem:
    """A config's batch on the device plus oracle-side weights of the experts
    it touches; inter_gs from the oracle's warmup (reading R8)."""

    def __init__(self, cfg, oracle_tokens=None):
        self.cfg = cfg
        x, ids, w = W.batch(cfg)
        self.x, self.ids, self.w = x, ids, w
        xw, idw, ww = W.batch(cfg, warmup=True)
        if oracle_tokens is None:
            experts = list(range(cfg.E))
        else:                   # oracle weights only for the experts the oracle will touch
            used = set(np.unique(ids.numpy()[oracle_tokens]).tolist()) | set(np.unique(idw.numpy()).tolist())
            experts = sorted(used)
        self.ow = OracleWeights(cfg, experts, DEV)
        self.dw = prep.MoeWeights.synthetic(cfg, DEV)
        # warmup: per-expert max|h| on the warmup batch, 2688/amax, fallback for experts without rows
        xwb = W.bf16_bits(xw)
        _, inter = O.moe_forward(xwb, self.ow.remap_ids(idw.numpy()), ww.numpy(), O.global_scale_bf16(xwb),
                                 **self.ow.oracle_kwargs(), inter_gs=None, intermediates=True)
        amax = inter["h_amax"]
        full = np.zeros(cfg.E, np.float32)
        full[self.ow.experts] = amax
        gmax = full.max()
        self.inter_gs = np.array([O.global_scale_from_amax(a if a > 0 else gmax) for a in full], np.float32)
        self.x_gs = O.global_scale_bf16(W.bf16_bits(x))

    def oracle(self, intermediates=False):
        return O.moe_forward(W.bf16_bits(self.x), self.ow.remap_ids(self.ids.numpy()), self.w.numpy(), self.x_gs,
                             **self.ow.oracle_kwargs(), inter_gs=self.inter_gs[self.ow.experts],
                             intermediates=intermediates)

    def device_inputs(self):
        return dict(x=self.x.to(DEV), topk_ids=self.ids.to(DEV), topk_weights=self.w.to(DEV),
                    x_gs=torch.tensor([self.x_gs], device=DEV), **self.dw.args(),
                    inter_gs=torch.from_numpy(self.inter_gs).to(DEV))

    def run(self, inputs=None, ws=None):
        cfg = self.cfg
        T = self.x.shape[0]
        inputs = inputs or self.device_inputs()
        ws = prep.workspace(T, cfg.k, cfg.E, cfg.H, cfg.I, DEV) if ws is None else ws
        out = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
        nvfp4_moe_forward(**inputs, out=out, workspace=ws)
        torch.cuda.synchronize()
        return out, ws


def check_output(out, ref):
    got = bf16_to_np(out)
    assert np.all(np.isfinite(got))
    err = row_rel_l2(got, ref)
    assert err.max() <= ROW_TOL, (err.max(), err.argmax())
    assert row_max_rel(got, ref).max() <= ROW_TOL
    assert cosine(got, ref) >= COS_TOL


def region(p, r):
    cfg = p.cfg
    T = p.x.shape[0]
    return nvfp4_moe_workspace_region(T, cfg.k, cfg.E, cfg.H, cfg.I, r)


def check_weights_bitexact(p, experts):
    """The device-quantised weights equal the oracle's for these experts."""
    cfg = p.cfg
    H, I = cfg.H, cfg.I
    for i, e in enumerate(experts):
        j = p.ow.experts.index(e)
        np.testing.assert_array_equal(p.dw.w13_codes[e].cpu().numpy(), p.ow.w13_codes[j])
        np.testing.assert_array_equal(p.dw.w13_gs[e].cpu().numpy(), p.ow.w13_gs[j])
        s13 = 2 * I * (H // 16)
        np.testing.assert_array_equal(
            from_mma_layout(p.dw.w13_scales[e * s13:(e + 1) * s13].cpu().numpy(), 2 * I, H), p.ow.w13_scales[j])
        np.testing.assert_array_equal(p.dw.w2_codes[e].cpu().numpy(), p.ow.w2_codes[j])
        assert p.dw.w2_gs[e].item() == p.ow.w2_gs[j]


@pytest.fixture(scope="module")
def tiny():
    return Problem(W.MOE_CONFIGS["tiny"])


def check_intermediates(p, ws, inter):
    """Inside the forward's workspace: inv and counts equal the oracle's
    routing; x's codes and scales at every slot's padded row are bit-exact;
    h codes (which depend on fp32 accumulation order) >= 99 % identical with
    every mismatch an adjacent code; the oracle's L2 GEMM fed the GPU's own h
    matches the GPU's y within 5e-3 per row."""
    cfg = p.cfg
    T, k, H, I = p.x.shape[0], cfg.k, cfg.H, cfg.I
    wsn = ws.cpu().numpy()
    route = O.route(p.ids.numpy(), cfg.E)
    o, n = region(p, 5)
    inv = wsn[o:o + n].view(np.int32)
    np.testing.assert_array_equal(inv, route["pos_padded"])
    o, n = region(p, 6)
    np.testing.assert_array_equal(wsn[o:o + n].view(np.int32), route["counts"])
    live = inv >= 0

    # x codes / scales at every slot's padded row: bit-exact
    xc, xs = O.quantize_bf16(W.bf16_bits(p.x), p.x_gs)
    o, n = region(p, 0)
    a_codes = wsn[o:o + n].reshape(-1, H // 2)
    o, n = region(p, 1)                             # row blocks (include/nvfp4moe.h, region 1)
    a_sc = from_rowblock_layout(wsn[o:o + n], a_codes.shape[0], H)
    tok = np.arange(T * k) // k
    np.testing.assert_array_equal(a_codes[inv[live]], xc[tok[live]])
    np.testing.assert_array_equal(a_sc[inv[live]], xs[tok[live]])

    # h codes: fp32 accumulation order may move a value across a rounding edge
    o, n = region(p, 2)
    h_codes = wsn[o:o + n].reshape(-1, I // 2)[inv[live]]
    o, n = region(p, 3)
    h_sc = from_mma_layout(wsn[o:o + n], a_codes.shape[0], I)[inv[live]]
    ref_codes = inter["h_codes"][live]
    ref_q = np.stack([ref_codes & 15, ref_codes >> 4], -1).reshape(-1, I)
    got_q = np.stack([h_codes & 15, h_codes >> 4], -1).reshape(-1, I)
    same = got_q == ref_q
    assert same.mean() >= 0.99, same.mean()
    mag = lambda c: np.where(c & 8, -(c & 7).astype(int), (c & 7).astype(int))
    assert np.all(np.abs(mag(got_q) - mag(ref_q))[~same] <= 1)
    assert (h_sc == inter["h_scales"][live]).mean() >= 0.99

    # staged: oracle L2 on the GPU's own h, per expert, against the GPU's y
    o, n = region(p, 4)
    y = wsn[o:o + n].view(np.uint16).reshape(T * k, H)
    y = (y.astype(np.uint32) << 16).view(np.float32)
    flat = p.ids.numpy().reshape(-1)
    yrow = np.where(live, route["offsets"][np.clip(flat, 0, cfg.E - 1)] + route["rank"], -1)
    live_idx = np.nonzero(live)[0]
    for e in range(cfg.E):
        sel = np.nonzero(flat[live_idx] == e)[0]          # positions among the live slots
        if sel.size == 0:
            continue
        j = p.ow.experts.index(e)
        ye = O.gemm(h_codes[sel], h_sc[sel], p.inter_gs[e], p.ow.w2_codes[j], p.ow.w2_scales[j],
                    p.ow.w2_gs[j:j + 1])
        err = row_rel_l2(y[yrow[live_idx[sel]]], ye)
        assert err.max() <= 5e-3, (e, err.max())


def test_tiny_end_to_end_and_intermediates(tiny):
    p = tiny
    check_weights_bitexact(p, range(p.cfg.E))
    out, ws = p.run()
    ref, inter = p.oracle(intermediates=True)
    check_output(out, ref)
    assert nvfp4_moe_get_error(ws) == 0
    check_intermediates(p, ws, inter)


def test_tiny_with_skipped_slots(tiny):
    p = tiny
    inputs = p.device_inputs()
    ids = p.ids.clone()
    ids[::3, 1] = -1
    inputs["topk_ids"] = ids.to(DEV)
    out, ws = p.run(inputs)
    ref = O.moe_forward(W.bf16_bits(p.x), ids.numpy(), p.w.numpy(), p.x_gs, **p.ow.oracle_kwargs(),
                        inter_gs=p.inter_gs)
    check_output(out, ref)
    assert nvfp4_moe_get_error(ws) == 0


def test_tiny_bad_ids_set_error_word(tiny):
    p = tiny
    inputs = p.device_inputs()
    ids = p.ids.clone()
    ids[5, 0] = p.cfg.E + 3
    inputs["topk_ids"] = ids.to(DEV)
    out, ws = p.run(inputs)
    assert nvfp4_moe_get_error(ws) == -8
    ids_skip = ids.numpy().copy()
    ids_skip[5, 0] = -1
    ref = O.moe_forward(W.bf16_bits(p.x), ids_skip, p.w.numpy(), p.x_gs, **p.ow.oracle_kwargs(),
                        inter_gs=p.inter_gs)
    check_output(out, ref)


def test_calibrate_matches_oracle_warmup(tiny):
    p = tiny
    cfg = p.cfg
    xw, idw, ww = W.batch(cfg, warmup=True)
    gs = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(xw.to(DEV), gs)
    ws = prep.workspace(xw.shape[0], cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    got = torch.empty(cfg.E, dtype=torch.float32, device=DEV)
    nvfp4_moe_calibrate(xw.to(DEV), idw.to(DEV), ww.to(DEV), gs, **p.dw.args(), inter_gs_out=got, workspace=ws)
    got = got.cpu().numpy()
    np.testing.assert_allclose(got, p.inter_gs, rtol=2e-6)


def test_cuda_graph_replay_with_new_inputs(tiny):
    """Capture once, replay with new x and topk ids of the same shape
    (page 1 "Phase 1": cudagraph-safe runner, pre-allocated buffers)."""
    p = tiny
    cfg = p.cfg
    T = p.x.shape[0]
    inputs = p.device_inputs()
    ws = prep.workspace(T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    out = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=DEV)
    nvfp4_moe_forward(**inputs, out=out, workspace=ws)          # eager call first (per-kernel attributes)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            nvfp4_moe_forward(**inputs, out=out, workspace=ws, stream=s)
    g2 = torch.Generator().manual_seed(99)
    x2 = torch.randn(T, cfg.H, generator=g2).to(torch.bfloat16)
    ids2 = torch.stack([torch.randperm(cfg.E, generator=g2)[:cfg.k] for _ in range(T)]).to(torch.int32)
    inputs["x"].copy_(x2.to(DEV))
    inputs["topk_ids"].copy_(ids2.to(DEV))
    g.replay()
    torch.cuda.synchronize()
    ref = O.moe_forward(W.bf16_bits(x2), ids2.numpy(), p.w.numpy(), p.x_gs, **p.ow.oracle_kwargs(),
                        inter_gs=p.inter_gs)
    check_output(out, ref)
    eager = torch.empty_like(out)
    nvfp4_moe_forward(**inputs, out=eager, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(eager, out)


@pytest.mark.parametrize("name", ["decode", "shared", "decode_shared", "tiny_shared"])
def test_full_size_configs(name):
    cfg = W.MOE_CONFIGS[name]
    p = Problem(cfg)
    check_weights_bitexact(p, [0, cfg.E - 1])
    out, ws = p.run()
    ref, inter = p.oracle(intermediates=True)
    check_output(out, ref)
    assert nvfp4_moe_get_error(ws) == 0
    if name == "decode":            # the full-size epilogue's h codes and the staged L2 as well
        check_intermediates(p, ws, inter)


def test_prefill_ep48_full_output():
    """Prefill-shaped routing on one expert-parallel slice (48 experts, top-6,
    T = 512, Zipf-skewed with 2 empty experts, heavy experts of several
    128-row m-tiles next to experts of a few rows): every output row against
    the oracle, and the intermediates inside the workspace."""
    cfg = W.MOE_CONFIGS["prefill_ep48"]
    p = Problem(cfg)
    counts = np.bincount(p.ids.numpy().ravel(), minlength=cfg.E)
    assert (counts == 0).sum() >= 2 and counts.max() > 256 and ((counts > 0) & (counts <= 32)).any()
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    ref, inter = p.oracle(intermediates=True)
    check_output(out, ref)
    check_intermediates(p, ws, inter)


def boundary_tokens(ids, E, k):
    """Tokens whose routed slots land where a full-size launch does something
    special: the heaviest expert's first row, the rows on both sides of its
    first 128-row and 256-row boundaries, a row of a middle m-tile and the
    last row of its last (partial) m-tile; the second heaviest expert's first
    row of its second m-tile and its last row; the first row of the expert
    with the fewest rows (one or two)."""
    flat = ids.reshape(-1)
    counts = np.bincount(flat[flat >= 0], minlength=E)
    order = np.argsort(-counts, kind="stable")

    def tok(e, r):
        return int(np.nonzero(flat == e)[0][min(r, counts[e] - 1)]) // k

    e0, e1 = int(order[0]), int(order[1])
    c0 = int(counts[e0])
    mid = ((c0 + 127) // 128 // 2) * 128 + 5
    picks = [tok(e0, r) for r in (0, 127, 128, 255, 256, mid, c0 - 1)]
    picks += [tok(e1, 128), tok(e1, int(counts[e1]) - 1)]
    emin = int(np.where(counts > 0, counts, np.iinfo(np.int64).max).argmin())
    picks.append(tok(emin, 0))
    return sorted(set(picks))


@pytest.mark.parametrize("name", ["prefill", "prefill_shared"])
def test_prefill_sampled_tokens(name):
    """384 experts, Zipf-skewed routing with empty experts: the whole batch on
    the GPU; through the oracle, the tokens at the launch's boundaries
    (boundary_tokens) and four random ones.  prefill_shared adds the shared
    expert as a 385th group that every token reaches (32 m-tiles)."""
    cfg = W.MOE_CONFIGS[name]
    ids = W.batch(cfg)[1].numpy()
    targeted = boundary_tokens(ids, cfg.E, cfg.k)
    tokens = np.unique(np.concatenate([targeted, np.random.default_rng(0).choice(cfg.T, 4, replace=False)]))
    p = Problem(cfg, oracle_tokens=tokens)
    route = O.route(p.ids.numpy(), cfg.E)
    assert (route["counts"] == 0).sum() >= 16                  # some experts are empty
    check_weights_bitexact(p, p.ow.experts[:2])
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    ref = O.moe_forward(W.bf16_bits(p.x[tokens]), p.ow.remap_ids(p.ids.numpy()[tokens]), p.w.numpy()[tokens],
                        p.x_gs, **p.ow.oracle_kwargs(), inter_gs=p.inter_gs[p.ow.experts])
    check_output(out[torch.from_numpy(tokens).to(DEV)], ref)
    # every routed row of the batch: inv matches the oracle's stable positions
    o, n = region(p, 5)
    np.testing.assert_array_equal(ws[o:o + n].cpu().numpy().view(np.int32), route["pos_padded"])


def test_forward_timed_matches_forward_eager_and_in_graph(tiny):
    """nvfp4_moe_forward_timed gives the same output as nvfp4_moe_forward and
    records six increasing timestamps, also when captured into a CUDA graph."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_forward_timed
    p = tiny
    cfg = p.cfg
    T = p.x.shape[0]
    inputs = p.device_inputs()
    ref, ws = p.run(inputs)
    for graph in (False, True):
        ev = [torch.cuda.Event(enable_timing=True, external=graph) for _ in range(6)]
        out = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
        if graph:
            for e in ev:
                e.record()
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    nvfp4_moe_forward_timed(**inputs, out=out, workspace=ws, events=ev, stream=s)
            g.replay()
        else:
            nvfp4_moe_forward_timed(**inputs, out=out, workspace=ws, events=ev)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        times = [ev[0].elapsed_time(e) for e in ev]
        assert all(b >= a for a, b in zip(times, times[1:])) and times[-1] > 0


# 12 experts, top-3, 1024 tokens: 256 routed rows per expert on average (two
# full m-tiles), so the grouped GEMMs run as pair tiles (clusters of two CTAs
# on 256-row tiles).
PAIRS = W.MoeConfig("pairs", E=12, k=3, T=1024, H=512, I=256, routing="zipf", outliers=True, warmup_T=256,
                    zipf_zero_tail=2)


def test_pair_tiles_end_to_end():
    """Pair tiles: experts with an odd number of 128-row m-tiles (the second
    CTA of the last pair has no rows), with one m-tile, with several, and
    empty experts; the whole output against the oracle."""
    p = Problem(PAIRS)
    counts = np.bincount(p.ids.numpy().ravel(), minlength=PAIRS.E)
    mt = (counts + 127) // 128
    assert (mt % 2 == 1).any() and (mt >= 4).any() and (counts == 0).any()
    assert PAIRS.T * PAIRS.k >= 256 * PAIRS.E
    check_weights_bitexact(p, range(PAIRS.E))
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, p.oracle())


# H = 384: the L2 tiles are 128 wide, so L1 and L2 run as two launches.
NARROW = W.MoeConfig("narrow", E=4, k=2, T=96, H=384, I=256, routing="softmax", outliers=False, warmup_T=64)


def test_unfused_narrow_hidden():
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_plan
    assert nvfp4_moe_plan(NARROW.T, NARROW.k, NARROW.E, NARROW.H, NARROW.I) == (False, 0)
    p = Problem(NARROW)
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, p.oracle())


def test_forward_computes_batch_global_scale(tiny):
    """x_gs = None: the forward computes 2688 / max|x| of the batch in its
    front launch (kept in workspace region 8), equal bit for bit to the
    oracle's global scale, and the output equals that of a call given the
    same scale explicitly."""
    p = tiny
    inputs = p.device_inputs()
    ref_out, ws = p.run(inputs)
    cfg = p.cfg
    T = p.x.shape[0]
    inputs_none = dict(inputs, x_gs=None)
    out = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
    nvfp4_moe_forward(**inputs_none, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert nvfp4_moe_get_error(ws) == 0
    o, n = region(p, 8)
    gs = ws[o:o + n].cpu().numpy().view(np.float32)[0]
    assert gs == O.global_scale_bf16(W.bf16_bits(p.x)) == p.x_gs
    assert torch.equal(out, ref_out)


EDGE = [
    W.MoeConfig("one_token", E=8, k=2, T=1, H=256, I=128, routing="softmax", outliers=False, warmup_T=64),
    W.MoeConfig("top32", E=64, k=32, T=16, H=256, I=128, routing="sigmoid", outliers=False, warmup_T=64),
    W.MoeConfig("e1024", E=1024, k=4, T=24, H=256, I=128, routing="softmax", outliers=True, warmup_T=64),
]


@pytest.mark.parametrize("cfg", EDGE, ids=[c.name for c in EDGE])
def test_edge_shapes_end_to_end(cfg):
    """One token; the largest top-k (32); the largest expert count (1024,
    most experts empty): the whole output against the oracle."""
    p = Problem(cfg)
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, p.oracle())


def test_prefill_pure_zipf_sampled_tokens():
    """The prefill batch with pure Zipf popularity (no empty expert, the
    heaviest expert ~3100 rows, one expert of a single row): the boundary
    tokens and two random ones through the oracle."""
    cfg = W.MOE_CONFIGS["prefill_zipf_pure"]
    ids = W.batch(cfg)[1].numpy()
    targeted = boundary_tokens(ids, cfg.E, cfg.k)
    tokens = np.unique(np.concatenate([targeted, np.random.default_rng(1).choice(cfg.T, 2, replace=False)]))
    p = Problem(cfg, oracle_tokens=tokens)
    route = O.route(p.ids.numpy(), cfg.E)
    assert (route["counts"] == 0).sum() == 0 and (route["counts"] == 1).sum() >= 1
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    ref = O.moe_forward(W.bf16_bits(p.x[tokens]), p.ow.remap_ids(p.ids.numpy()[tokens]), p.w.numpy()[tokens],
                        p.x_gs, **p.ow.oracle_kwargs(), inter_gs=p.inter_gs[p.ow.experts])
    check_output(out[torch.from_numpy(tokens).to(DEV)], ref)


def test_bounded_wait_times_out_and_context_survives(tiny):
    """Failure detection without a fault: the fused launch's device wait on a
    counter that nothing raises gives up after its bound and reports
    NVFP4_ERR_TIMEOUT; a satisfied wait reports nothing; the context is still
    usable afterwards (a forward matches the oracle)."""
    import time
    from nvfp4_moe_expert_topk_b200 import nvfp4_debug_bounded_wait
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    nvfp4_debug_bounded_wait(flag, 1, err)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert err.item() == -7 and 1.5 < waited < 30.0
    flag.fill_(3)
    err.zero_()
    nvfp4_debug_bounded_wait(flag, 3, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    out, ws = tiny.run()
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, tiny.oracle())


# 16 experts, top-4, 768 tokens, Zipf-skewed: 3072 routed rows, so the plan
# puts the full m-tile pairs of experts with two or more m-tiles on pair
# tiles (their own L1 and L2 launches) and the rest on the fused 1-CTA
# launch.  m-tiles per expert: 6, 4, 3, 3, 2, 2, 2, 2, six of 1, two empty.
SPLIT = W.MoeConfig("split", E=16, k=4, T=768, H=512, I=256, routing="zipf", outliers=True, warmup_T=128,
                    zipf_zero_tail=2)


def expected_tile_tables(counts, pair_mode):
    """The tile tables the routing must write, from the plan's rule (include/
    nvfp4moe.h, nvfp4_moe_plan): m-tiles in expert order, 128 rows each, the
    last one partial; pairs of consecutive m-tiles; the light list."""
    mtiles, pairs, light = [], [], []
    row, yrow = 0, 0
    for e, c in enumerate(counts):
        tiles = (int(c) + 127) // 128
        first = len(mtiles)
        for i in range(tiles):
            mtiles.append((e, row + 128 * i, min(128, int(c) - 128 * i), yrow + 128 * i))
        if pair_mode == 1:
            npair = tiles // 2 if tiles >= 2 else 0
        elif pair_mode == 2:
            npair = (tiles + 1) // 2
        else:
            npair = 0
        for i in range(npair):
            pairs.append((first + 2 * i, first + 2 * i + 1 if 2 * i + 1 < tiles else -1))
        light += list(range(first + min(2 * npair, tiles), first + tiles))
        row += 128 * tiles
        yrow += int(c)
    return np.array(mtiles, np.int32).reshape(-1, 4), np.array(pairs, np.int32).reshape(-1, 2), \
        np.array(light, np.int32)


def check_tile_tables(p, ws, pair_mode):
    cfg = p.cfg
    counts = np.bincount(p.ids.numpy().ravel()[p.ids.numpy().ravel() >= 0], minlength=cfg.E)
    mt, pr, lt = expected_tile_tables(counts, pair_mode)
    wsn = ws.cpu().numpy()
    o, n = region(p, 12)
    hdr = wsn[o:o + n].view(np.int32)
    assert (hdr[1], hdr[2], hdr[6]) == (len(mt), len(pr), len(lt))
    o, n = region(p, 9)
    np.testing.assert_array_equal(wsn[o:o + n].view(np.int32).reshape(-1, 4)[:len(mt)], mt)
    o, n = region(p, 10)
    np.testing.assert_array_equal(wsn[o:o + n].view(np.int32).reshape(-1, 2)[:len(pr)], pr)
    o, n = region(p, 11)
    np.testing.assert_array_equal(wsn[o:o + n].view(np.int32)[:len(lt)], lt)


def test_split_pair_and_light_tiles_end_to_end():
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_plan
    assert nvfp4_moe_plan(SPLIT.T, SPLIT.k, SPLIT.E, SPLIT.H, SPLIT.I) == (True, 1)
    p = Problem(SPLIT)
    counts = np.bincount(p.ids.numpy().ravel(), minlength=SPLIT.E)
    mt = (counts + 127) // 128
    assert ((mt >= 2) & (mt % 2 == 0)).any() and ((mt >= 3) & (mt % 2 == 1)).any() and (mt == 1).any()
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    ref, inter = p.oracle(intermediates=True)
    check_output(out, ref)
    check_intermediates(p, ws, inter)
    check_tile_tables(p, ws, 1)


@pytest.mark.parametrize("name,mode", [("decode", 0), ("prefill_ep48", 1)])
def test_tile_tables_of_full_size_routing(name, mode):
    """The routing's tile tables on the decode batch (every m-tile light) and
    on the 48-expert prefill slice (pairs for its heavy experts)."""
    cfg = W.MOE_CONFIGS[name]
    x, ids, w = W.batch(cfg)
    p = Problem.__new__(Problem)               # routing only: no oracle weights needed
    p.cfg, p.x, p.ids, p.w = cfg, x, ids, w
    dw = prep.MoeWeights.synthetic(cfg, DEV)
    ws = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    nvfp4_moe_forward(x.to(DEV), ids.to(DEV), w.to(DEV), None, **dw.args(),
                      inter_gs=torch.ones(cfg.E, device=DEV), out=out, workspace=ws)
    torch.cuda.synchronize()
    assert nvfp4_moe_get_error(ws) == 0
    check_tile_tables(p, ws, mode)
    route = O.route(ids.numpy(), cfg.E)
    o, n = region(p, 5)
    np.testing.assert_array_equal(ws[o:o + n].cpu().numpy().view(np.int32), route["pos_padded"])


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill_ep48"])
def test_forward_on_prequantised_rows_equals_forward(name):
    """nvfp4_moe_forward_quantized on the codes and row-major scales that
    nvfp4_quantize makes from x with x_gs gives nvfp4_moe_forward's output on
    x with x_gs bit for bit (the front only permutes the given rows)."""
    from nvfp4_moe_expert_topk_b200 import NVFP4_SCALES_ROWMAJOR, nvfp4_moe_forward_quantized, nvfp4_quantize
    cfg = W.MOE_CONFIGS[name]
    x, ids, w = W.batch(cfg)
    dw = prep.MoeWeights.synthetic(cfg, DEV)
    xd, idd, wd = x.to(DEV), ids.to(DEV), w.to(DEV)
    gs = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(xd, gs)
    inter = torch.full((cfg.E,), 40.0, dtype=torch.float32, device=DEV)
    ws = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    ref = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    nvfp4_moe_forward(xd, idd, wd, gs, **dw.args(), inter_gs=inter, out=ref, workspace=ws)
    codes = torch.empty(cfg.T, cfg.H // 2, dtype=torch.uint8, device=DEV)
    scales = torch.empty(cfg.T, cfg.H // 16, dtype=torch.uint8, device=DEV)
    nvfp4_quantize(xd, gs, codes, scales, NVFP4_SCALES_ROWMAJOR)
    out = torch.full_like(ref, float("nan"))
    ws2 = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    nvfp4_moe_forward_quantized(codes, scales, idd, wd, gs, **dw.args(), inter_gs=inter, out=out, workspace=ws2)
    torch.cuda.synchronize()
    assert nvfp4_moe_get_error(ws2) == 0
    assert torch.isfinite(out.float()).all() and torch.equal(out, ref)


def test_cuda_graph_replay_split_plan_with_new_inputs():
    """Pair mode 1 captured in a CUDA graph (the pair launch triggering its
    dependent early, the 1-CTA launch claiming tiles, the counters reset by
    the front each step): replays with new x and new routing equal eager
    calls bit for bit, and the oracle within the bar."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_plan
    cfg = SPLIT
    assert nvfp4_moe_plan(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I) == (True, 1)
    p = Problem(cfg)
    inputs = p.device_inputs()
    inputs["x_gs"] = None                       # the batch's global scale inside the graph as well
    ws = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    nvfp4_moe_forward(**inputs, out=out, workspace=ws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            nvfp4_moe_forward(**inputs, out=out, workspace=ws, stream=s)
    for seed in (5, 6):
        rng = torch.Generator().manual_seed(seed)
        x2 = torch.randn(cfg.T, cfg.H, generator=rng).to(torch.bfloat16)
        ids2 = W.routing(cfg, cfg.T, seed=300 + seed)[0]
        inputs["x"].copy_(x2.to(DEV))
        inputs["topk_ids"].copy_(ids2.to(DEV))
        g.replay()
        torch.cuda.synchronize()
        assert nvfp4_moe_get_error(ws) == 0
        eager = torch.empty_like(out)
        ws2 = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
        nvfp4_moe_forward(**inputs, out=eager, workspace=ws2)
        torch.cuda.synchronize()
        assert torch.equal(eager, out)
        xb = W.bf16_bits(x2)
        ref = O.moe_forward(xb, ids2.numpy(), p.w.numpy(), O.global_scale_bf16(xb), **p.ow.oracle_kwargs(),
                            inter_gs=p.inter_gs)
        check_output(out, ref)


def test_empty_batch_runs_nothing():
    """T = 0 through the Python API: the forward, the pre-quantised forward
    and the calibration accept empty tensors (NULL batch pointers); the
    forward writes nothing and sets no error, and the calibration of an
    empty warmup batch gives every expert the global scale of amax = 0."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_calibrate, nvfp4_moe_forward_quantized, prep
    cfg = W.MOE_CONFIGS["tiny"]
    p = Problem(cfg)
    inputs = p.device_inputs()
    H = cfg.H
    ws = prep.workspace(0, cfg.k, cfg.E, H, cfg.I, DEV)
    x0 = torch.empty(0, H, dtype=torch.bfloat16, device=DEV)
    ids0 = torch.empty(0, cfg.k, dtype=torch.int32, device=DEV)
    w0 = torch.empty(0, cfg.k, dtype=torch.float32, device=DEV)
    out0 = torch.empty(0, H, dtype=torch.bfloat16, device=DEV)
    args = {k: v for k, v in inputs.items() if k not in ("x", "topk_ids", "topk_weights", "x_gs")}
    nvfp4_moe_forward(x0, ids0, w0, None, **args, out=out0, workspace=ws)
    x_gs = torch.ones(1, dtype=torch.float32, device=DEV)
    nvfp4_moe_forward_quantized(torch.empty(0, H // 2, dtype=torch.uint8, device=DEV),
                                torch.empty(0, H // 16, dtype=torch.uint8, device=DEV), ids0, w0, x_gs, **args,
                                out=out0, workspace=ws)
    igs = torch.full((cfg.E,), -1.0, dtype=torch.float32, device=DEV)
    cal = {k: v for k, v in args.items() if k != "inter_gs"}
    nvfp4_moe_calibrate(x0, ids0, w0, x_gs, **cal, inter_gs_out=igs, workspace=ws)
    torch.cuda.synchronize()
    assert nvfp4_moe_get_error(ws) == 0
    assert bool((igs == float(O.global_scale_from_amax(0.0))).all()), igs


def random_config(seed):
    """A small MoE shape drawn from the seed: 2-40 experts, top-1..8, 1-1024
    tokens, H in 128..512, I in 128..384, softmax or Zipf routing (some
    experts empty), with or without outlier channels.  Large enough batches
    reach the pair plans (R >= 2048, or R >= 256 E with H % 256 == 0), H not
    a multiple of 256 the two-launch plan."""
    rng = np.random.default_rng(1000 + seed)
    E = int(rng.integers(2, 41))
    k = int(rng.integers(1, min(8, E) + 1))
    T = int(rng.choice([1, 7, 64, 129, 300, 600, 1024]))
    H = int(rng.choice([128, 256, 256, 384, 512, 512]))
    I = int(rng.choice([128, 256, 384]))
    routing = str(rng.choice(["softmax", "zipf"]))
    tail = int(min(2, E - k))
    return W.MoeConfig(f"random{seed}", E=E, k=k, T=T, H=H, I=I, routing=routing, outliers=bool(rng.integers(2)),
                       warmup_T=64, zipf_zero_tail=tail)


@pytest.mark.parametrize("seed", range(48))
def test_random_configs_match_oracle(seed):
    """Every output row of a randomly drawn small config against the oracle,
    whatever plan the forward picks for it."""
    cfg = random_config(seed)
    p = Problem(cfg)
    out, ws = p.run()
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, p.oracle())


@pytest.mark.parametrize("seed", range(16))
def test_random_configs_with_shared_experts_and_skipped_slots(seed):
    """Seeded random configs with one or two shared experts folded in (the
    last slots, weight 1) and about a fifth of the routed slots skipped
    (id -1): every output row against the oracle."""
    base = random_config(100 + seed)
    rng = np.random.default_rng(500 + seed)
    shared = int(rng.integers(1, 3))
    cfg = W.MoeConfig(f"random_shared{seed}", E=base.E + shared, k=base.k + shared, T=base.T, H=base.H, I=base.I,
                      routing="softmax", outliers=base.outliers, warmup_T=64, shared=shared)
    p = Problem(cfg)
    ids = p.ids.clone()
    skip = torch.from_numpy(rng.random((ids.shape[0], cfg.k - shared)) < 0.2)
    ids[:, :cfg.k - shared][skip] = -1
    inputs = p.device_inputs()
    inputs["topk_ids"] = ids.to(DEV)
    out, ws = p.run(inputs)
    ref = O.moe_forward(W.bf16_bits(p.x), p.ow.remap_ids(ids.numpy()), p.w.numpy(), p.x_gs,
                        **p.ow.oracle_kwargs(), inter_gs=p.inter_gs[p.ow.experts])
    assert nvfp4_moe_get_error(ws) == 0
    check_output(out, ref)
