"""GPU parity of the top-k router (nvfp4_moe_topk) against the oracle's
oracle_topk: ids bit-exact (ties to the lower expert id), weights within
rtol 1e-5.  The bound: the kernel evaluates each exp or sigmoid in fp32
(a few ulp), sums at most 32 positive terms in fp32 (relative error below
31 * 2^-24) and rounds one division; together under 3e-6 of the weight."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_moe_expert_topk_b200 import (NVFP4_SCORING_SIGMOID, NVFP4_SCORING_SOFTMAX, nvfp4_moe_topk,
                                        nvfp4_moe_topk_shared)

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCORING = {"softmax": NVFP4_SCORING_SOFTMAX, "sigmoid": NVFP4_SCORING_SIGMOID}


def run_topk(logits, k, scoring):
    T = logits.shape[0]
    ids = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device=DEV)
    nvfp4_moe_topk(torch.from_numpy(logits).to(DEV), k, ids, w, SCORING[scoring])
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def check(logits, k, scoring):
    ids, w = run_topk(logits, k, scoring)
    rid, rw = O.topk(logits, k, scoring)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-5, atol=0)


@pytest.mark.parametrize("T,E,k,scoring", [
    (1, 8, 1, "softmax"),
    (37, 48, 6, "sigmoid"),       # 48 experts, top-6 (one expert-parallel shard of 384)
    (4096, 384, 6, "sigmoid"),    # 384 experts, top-6, a full prefill batch
    (513, 384, 8, "softmax"),
    (100, 1024, 32, "softmax"),   # largest E and k
    (64, 33, 5, "sigmoid"),       # E not a multiple of 32
    (9, 6, 6, "softmax"),         # k == E
])
def test_topk_matches_oracle(T, E, k, scoring):
    rng = np.random.default_rng(T * 31 + E)
    logits = rng.normal(0, 1.5, (T, E)).astype(np.float32)
    check(logits, k, scoring)


@pytest.mark.parametrize("scoring", ["softmax", "sigmoid"])
def test_topk_ties_go_to_lower_id(scoring):
    rng = np.random.default_rng(5)
    logits = (rng.integers(-3, 4, (300, 384)) / 4.0).astype(np.float32)   # many equal logits per row
    logits[0] = 1.0                                                      # all equal
    logits[1] = 0.0
    logits[1, ::2] = -0.0                                                # -0 and +0 are equal
    logits[2, 383] = logits[2, 200] = logits[2, 7] = 50.0                # tie at the top across lanes
    check(logits, 6, scoring)
    ids, _ = run_topk(logits, 6, scoring)
    assert ids[0].tolist() == list(range(6)) and ids[1].tolist() == list(range(6))
    assert ids[2, :3].tolist() == [7, 200, 383]


def test_topk_empty_batch():
    ids = torch.empty((0, 6), dtype=torch.int32, device=DEV)
    w = torch.empty((0, 6), dtype=torch.float32, device=DEV)
    nvfp4_moe_topk(torch.empty((0, 384), dtype=torch.float32, device=DEV), 6, ids, w, NVFP4_SCORING_SIGMOID)
    torch.cuda.synchronize()


def test_topk_feeds_forward():
    """Router output drives the MoE forward: the device router's ids equal the
    oracle router's, and the forward on them matches the oracle forward."""
    from test_gpu_moe import Problem, check_output
    from nvfp4_moe_expert_topk_b200 import workloads as W
    cfg = W.MOE_CONFIGS["tiny"]
    p = Problem(cfg)
    rng = np.random.default_rng(11)
    logits = rng.normal(0, 1, (p.x.shape[0], cfg.E)).astype(np.float32)
    ids, w = run_topk(logits, cfg.k, "softmax")
    rid, rw = O.topk(logits, cfg.k, "softmax")
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-5, atol=0)
    p.ids, p.w = torch.from_numpy(ids), torch.from_numpy(w)
    out, _ = p.run()
    check_output(out, p.oracle())


@pytest.mark.parametrize("T,E,k,ns,scoring", [
    (64, 48, 6, 1, "sigmoid"),    # the decode shard with the shared expert folded in
    (300, 384, 6, 2, "softmax"),
    (7, 40, 30, 2, "softmax"),    # k + num_shared = 32: every lane writes a slot
    (5, 1023, 8, 1, "sigmoid"),   # E + num_shared = 1024
])
def test_topk_shared_matches_oracle(T, E, k, ns, scoring):
    rng = np.random.default_rng(T + 7 * E)
    logits = rng.normal(0, 1.5, (T, E)).astype(np.float32)
    ids = torch.full((T, k + ns), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k + ns), float("nan"), dtype=torch.float32, device=DEV)
    nvfp4_moe_topk_shared(torch.from_numpy(logits).to(DEV), k, ns, ids, w, SCORING[scoring])
    torch.cuda.synchronize()
    rid, rw = O.topk(logits, k, scoring, num_shared=ns)
    np.testing.assert_array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=1e-5, atol=0)
    assert (w[:, k:] == 1.0).all()


def test_topk_shared_feeds_forward():
    """Router with the shared expert folded in drives the forward over the
    routed experts plus the shared one: ids bit-exact against the oracle
    router, the output against the oracle forward on them."""
    from test_gpu_moe import Problem, check_output
    from nvfp4_moe_expert_topk_b200 import workloads as W
    cfg = W.MOE_CONFIGS["tiny_shared"]
    p = Problem(cfg)
    rng = np.random.default_rng(12)
    T, Er, k = p.x.shape[0], cfg.E - cfg.shared, cfg.k - cfg.shared
    logits = rng.normal(0, 1, (T, Er)).astype(np.float32)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    nvfp4_moe_topk_shared(torch.from_numpy(logits).to(DEV), k, cfg.shared, ids, w, NVFP4_SCORING_SOFTMAX)
    torch.cuda.synchronize()
    rid, rw = O.topk(logits, k, "softmax", num_shared=cfg.shared)
    np.testing.assert_array_equal(ids.cpu().numpy(), rid)
    p.ids, p.w = ids.cpu(), w.cpu()
    out, _ = p.run()
    check_output(out, p.oracle())


@pytest.mark.parametrize("seed", range(24))
def test_topk_random_shapes(seed):
    """Seeded random T (1-2000), E (1-1024), k (1-min(32, E)), scoring and
    logit scale, a quarter of the logits quantised to a coarse grid so that
    ties occur: ids bit-exact, weights within the bound."""
    rng = np.random.default_rng(4000 + seed)
    E = int(rng.integers(1, 1025))
    k = int(rng.integers(1, min(32, E) + 1))
    T = int(rng.integers(1, 2001))
    scoring = str(rng.choice(["softmax", "sigmoid"]))
    logits = rng.normal(0, float(rng.choice([0.3, 1.5, 6.0])), (T, E)).astype(np.float32)
    coarse = rng.random((T, E)) < 0.25
    logits[coarse] = np.round(logits[coarse] * 2) / 2
    check(logits, k, scoring)
