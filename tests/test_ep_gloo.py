"""Expert parallelism on gloo ranks (CPU; two ranks, and four for a few
scenarios): each rank owns an equal share of the experts and its own batch; the dispatch / per-rank experts / combine result
equals the single-process oracle on the union batch with the union's global
scale.  The per-rank expert computation here is the oracle (the library runs
only on a GPU); the exchange logic is the product's (ep.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from helpers import OracleWeights
from nvfp4_moe_expert_topk_b200 import workloads as W
from nvfp4_moe_expert_topk_b200.ep import ExpertParallelMoE, global_scale_from_amax

CFG = W.MoeConfig("ep_tiny", E=8, k=2, T=48, H=256, I=128, routing="softmax", outliers=False, warmup_T=64)
# the same routed experts plus one shared expert (global id 8, slot 2, weight 1)
CFG_SHARED = W.MoeConfig("ep_tiny_shared", E=9, k=3, T=48, H=256, I=128, routing="softmax", outliers=False,
                         warmup_T=64, shared=1)
WORLD = 2


def config(scenario):
    return CFG_SHARED if scenario.endswith("shared") else CFG


def rank_tokens(r, scenario):
    if scenario.endswith("empty_rank") and r == 1:
        return 0                                               # a rank with no tokens this step
    return CFG.T + 8 * r                                       # ranks hold different batch sizes


def rank_batch(r, scenario, world=WORLD):
    T = rank_tokens(r, scenario)
    x = W.activations(T, CFG.H, seed=100 + r)
    ids, w = W.routing(config(scenario), T, seed=200 + r)
    if scenario == "one_sided":                                # every slot on rank 0's experts
        ids = ids % (CFG.E // world)
    if scenario == "skips":
        ids[::5, 1] = -1                                       # skipped slots travel as -1
    return x, ids, w


def inter_gs_all(cfg):
    xw, idw, ww = W.batch(cfg, warmup=True)
    ow = OracleWeights(cfg, range(cfg.E), "cpu")
    xb = W.bf16_bits(xw)
    _, inter = O.moe_forward(xb, idw.numpy(), ww.numpy(), O.global_scale_bf16(xb), **ow.oracle_kwargs(),
                             inter_gs=None, intermediates=True)
    amax = inter["h_amax"]
    return np.array([O.global_scale_from_amax(a if a > 0 else amax.max()) for a in amax], np.float32)


def worker(rank, port, scenario, world=WORLD):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = config(scenario)
        El = CFG.E // world                                    # routed experts per rank
        shared = list(range(CFG.E, cfg.E))                     # replicated on every rank
        local = list(range(rank * El, (rank + 1) * El)) + shared
        ow = OracleWeights(cfg, local, "cpu")
        igs = inter_gs_all(cfg)

        def experts_fn(x, local_ids, w, gs):
            if isinstance(x, tuple):                           # NVFP4 rows: codes, row-major scales
                out = O.moe_forward(None, local_ids.numpy(), w.numpy(), gs, **ow.oracle_kwargs(),
                                    inter_gs=igs[local], x_codes=x[0].numpy(), x_scales=x[1].numpy())
            else:
                out = O.moe_forward(W.bf16_bits(x), local_ids.numpy(), w.numpy(), gs, **ow.oracle_kwargs(),
                                    inter_gs=igs[local])
            return torch.from_numpy(out)

        def quantize_fn(x, gs):
            c, sc = O.quantize_bf16(W.bf16_bits(x), gs) if x.shape[0] else \
                (np.zeros((0, CFG.H // 2), np.uint8), np.zeros((0, CFG.H // 16), np.uint8))
            return torch.from_numpy(np.ascontiguousarray(c)), torch.from_numpy(np.ascontiguousarray(sc))

        ep = ExpertParallelMoE(CFG.E, amax_fn=lambda x: O.amax_bf16(W.bf16_bits(x)), experts_fn=experts_fn,
                               num_shared=len(shared), quantize_fn=quantize_fn if "nvfp4" in scenario else None)
        x, ids, w = rank_batch(rank, scenario, world)
        got = ep.forward(x, ids, w, out_dtype=torch.float32).numpy()

        # reference: one process, all experts, the union batch
        xs, idss, ws = zip(*(rank_batch(r, scenario, world) for r in range(world)))
        xu, idu, wu = torch.cat(xs), torch.cat(idss), torch.cat(ws)
        gs = global_scale_from_amax(max(O.amax_bf16(W.bf16_bits(xr)) if xr.numel() else 0.0 for xr in xs))
        assert gs == O.global_scale_bf16(W.bf16_bits(xu))
        owa = OracleWeights(cfg, range(cfg.E), "cpu")
        ref = O.moe_forward(W.bf16_bits(xu), idu.numpy(), wu.numpy(), gs, **owa.oracle_kwargs(), inter_gs=igs)
        lo = sum(rank_tokens(r, scenario) for r in range(rank))
        ref = ref[lo:lo + x.shape[0]]
        assert got.shape == ref.shape
        if ref.size:
            np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("scenario", ["plain", "one_sided", "skips", "shared", "empty_rank", "nvfp4",
                                      "nvfp4_shared", "nvfp4_empty_rank"])
def test_expert_parallel_two_ranks(scenario):
    mp.start_processes(worker, args=(free_port(), scenario), nprocs=WORLD, start_method="spawn")


@pytest.mark.parametrize("scenario", ["plain", "nvfp4_shared", "one_sided"])
def test_expert_parallel_four_ranks(scenario):
    """Two experts per rank: every token's slots spread over up to four ranks
    (one_sided: all on rank 0's two experts)."""
    mp.start_processes(worker, args=(free_port(), scenario, 4), nprocs=4, start_method="spawn")


def test_plan_rewrites_ids_per_rank():
    """The dispatch plan on its own: each destination gets exactly the tokens
    with a slot there, ids rewritten to that rank's local range, -1 elsewhere."""
    class Fake(ExpertParallelMoE):
        def __init__(self):
            self.world, self.rank, self.E, self.El = 4, 0, 16, 4
    ids = torch.tensor([[0, 5], [15, 14], [-1, 3], [8, 9]])
    tokens, local = Fake().plan(ids)
    assert [t.tolist() for t in tokens] == [[0, 2], [0], [3], [1]]
    assert local[0].tolist() == [[0, -1], [-1, 3]]
    assert local[1].tolist() == [[-1, 1]]
    assert local[2].tolist() == [[0, 1]]
    assert local[3].tolist() == [[3, 2]]


def test_plan_keeps_shared_slots_home():
    """Shared-expert slots (ids >= E) are served on the token's own rank as
    local ids El + (id - E); every token of the rank goes to itself."""
    class Fake(ExpertParallelMoE):
        def __init__(self, rank):
            self.world, self.rank, self.E, self.El, self.num_shared = 4, rank, 16, 4, 2
    ids = torch.tensor([[0, 5, 16, 17], [15, 14, 16, 17], [-1, 3, 16, -1]])
    tokens, local = Fake(2).plan(ids)
    assert [t.tolist() for t in tokens] == [[0, 2], [0], [0, 1, 2], [1]]
    assert local[0].tolist() == [[0, -1, -1, -1], [-1, 3, -1, -1]]
    assert local[2].tolist() == [[-1, -1, 4, 5], [-1, -1, 4, 5], [-1, -1, 4, -1]]
    assert local[3].tolist() == [[3, 2, -1, -1]]
