"""Seeded synthetic workloads for the NVFP4 routed-expert MoE chain.

This module only draws inputs: activations, router outputs (top-k ids and
weights) and bf16 weights.  It contains none of the chain's arithmetic (no
quantisation, no GEMM, no SiLU, no permutation); both the CUDA path and the
CPU oracle consume what it produces.

Shapes follow the pages ("nvfp4-megamoe-kernel / CURRENT_BUG.md"):
hidden 7168, expert intermediate 3072 (page 3, "Architecture Notes"),
384 routed experts with top-6, 48 per expert-parallel rank (page 1,
"Config values"; page 3, "Architecture Notes"), a shared expert run as a
one-group chain (page 1, "Phase 1"), and the MLA projections run as separate
NVFP4 GEMMs (page 1, "Phase 2", option 1; sizes from page 1, "Config values").
The pages use real DeepSeek-V4 checkpoint weights; these stand in for them
with N(0, 0.02) weights and N(0, 1) activations.

Seeds: x 0, warmup x 1, router 4 (warmup router 14), outlier channels 5,
expert-popularity permutation 6, W13 of expert e 1000+e, W2 of expert e 2000+e,
MLA weights 3000+i.
"""
from dataclasses import dataclass, field
from typing import Optional

import torch

SEED_X, SEED_X_WARMUP = 0, 1
SEED_ROUTER, SEED_ROUTER_WARMUP = 4, 14
SEED_OUTLIER, SEED_ZIPF_PERM = 5, 6
SEED_W13, SEED_W2, SEED_MLA = 1000, 2000, 3000
SEED_LOGITS = 7
WEIGHT_STD = 0.02


@dataclass(frozen=True)
class MoeConfig:
    name: str
    E: int
    k: int
    T: int
    H: int
    I: int
    routing: str            # "softmax" | "sigmoid" | "zipf" | "single"
    outliers: bool
    warmup_T: int           # tokens in the warmup batch that fixes inter_gs
    zipf_s: float = 1.1
    zipf_zero_tail: int = 16
    # the last `shared` of the E experts are shared experts: every token runs
    # them with weight 1 in its last `shared` of the k slots (the routed
    # draw picks k - shared of the first E - shared experts)
    shared: int = 0


MOE_CONFIGS = {
    "tiny": MoeConfig("tiny", E=8, k=2, T=64, H=256, I=128, routing="softmax", outliers=False, warmup_T=64),
    "shared": MoeConfig("shared", E=1, k=1, T=256, H=7168, I=3072, routing="single", outliers=True, warmup_T=256),
    "decode": MoeConfig("decode", E=48, k=6, T=64, H=7168, I=3072, routing="sigmoid", outliers=False, warmup_T=64),
    "prefill": MoeConfig("prefill", E=384, k=6, T=4096, H=7168, I=3072, routing="zipf", outliers=True, warmup_T=16),
    # the prefill batch with pure Zipf popularity (no expert forced empty)
    "prefill_zipf_pure": MoeConfig("prefill_zipf_pure", E=384, k=6, T=4096, H=7168, I=3072, routing="zipf",
                                   outliers=True, warmup_T=16, zipf_zero_tail=0),
    # prefill-shaped (64 routed rows per expert on average, Zipf-skewed) on one
    # expert-parallel slice: small enough to profile and to check in full
    "prefill_ep48": MoeConfig("prefill_ep48", E=48, k=6, T=512, H=7168, I=3072, routing="zipf", outliers=True,
                              warmup_T=64, zipf_zero_tail=2),
    # the prefill batch and routing with a 128-wide expert intermediate:
    # the front (global scale, routing, quantise + permute of x) is exactly
    # the prefill's, the weights are 1/24 of its (a small profiling case)
    "prefill_front": MoeConfig("prefill_front", E=384, k=6, T=4096, H=7168, I=128, routing="zipf", outliers=True,
                               warmup_T=16),
    # the decode batch with the shared expert folded in as a 49th group
    # (page 1 "Phase 1": the shared expert is the routed chain with one
    # expert and no routing; same H and I as a routed expert)
    "decode_shared": MoeConfig("decode_shared", E=49, k=7, T=64, H=7168, I=3072, routing="sigmoid",
                               outliers=False, warmup_T=64, shared=1),
    "prefill_shared": MoeConfig("prefill_shared", E=385, k=7, T=4096, H=7168, I=3072, routing="zipf",
                                outliers=True, warmup_T=16, shared=1),
    "tiny_shared": MoeConfig("tiny_shared", E=9, k=3, T=64, H=256, I=128, routing="softmax", outliers=False,
                             warmup_T=64, shared=1),
}


@dataclass(frozen=True)
class GemmConfig:
    name: str
    M: int
    N: int
    K: int
    seg_end: tuple = field(default=())     # dual global scales: row ends of each B segment


MLA_GEMMS = {
    # fused_wqa_wkv: q_a [1536, 7168] stacked with kv [512, 7168]; one global scale per half
    "wqa_wkv": GemmConfig("wqa_wkv", M=2048, N=2048, K=7168, seg_end=(1536, 2048)),
    # q_b: [128 heads x 512, q_lora_rank 1536]
    "q_b": GemmConfig("q_b", M=2048, N=65536, K=1536, seg_end=(65536,)),
    # o_b: [hidden 7168, 8192]
    "o_b": GemmConfig("o_b", M=2048, N=7168, K=8192, seg_end=(7168,)),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def activations(T: int, H: int, seed: int = SEED_X, outliers: bool = False) -> torch.Tensor:
    """x ~ N(0,1) in fp32, cast to bf16; with outliers, the first floor(0.01*H)
    channels of a seeded permutation are scaled by 20 before the cast."""
    x = torch.randn(T, H, generator=_gen(seed), dtype=torch.float32)
    if outliers:
        ch = torch.randperm(H, generator=_gen(SEED_OUTLIER))[: int(0.01 * H)]
        x[:, ch] *= 20.0
    return x.to(torch.bfloat16)


def _renorm(w: torch.Tensor) -> torch.Tensor:
    return (w / w.sum(dim=-1, keepdim=True)).to(torch.float32).contiguous()


def zipf_popularity(E: int, s: float, zero_tail: int) -> torch.Tensor:
    """Expert popularity: p(rank r) ~ r^-s with the `zero_tail` least popular
    ranks set to zero, mapped to expert ids by a seeded permutation."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    if zero_tail:
        p[E - zero_tail:] = 0.0
    p = p / p.sum()
    perm = torch.randperm(E, generator=_gen(SEED_ZIPF_PERM))
    pe = torch.empty(E, dtype=torch.float64)
    pe[perm] = p
    return pe


def routing(cfg: MoeConfig, T: Optional[int] = None, seed: int = SEED_ROUTER):
    """Top-k expert ids [T, k] int32 (descending score) and weights [T, k] fp32;
    with shared experts, the routed slots then one slot per shared expert
    (id E - shared + i, weight 1)."""
    T = cfg.T if T is None else T
    ids, w = _routed(cfg, T, _gen(seed), cfg.E - cfg.shared, cfg.k - cfg.shared)
    if cfg.shared:
        sid = torch.arange(cfg.E - cfg.shared, cfg.E, dtype=torch.int32).expand(T, cfg.shared)
        ids = torch.cat([ids, sid], dim=1).contiguous()
        w = torch.cat([w, torch.ones(T, cfg.shared, dtype=torch.float32)], dim=1).contiguous()
    return ids, w


def _routed(cfg: MoeConfig, T: int, g: torch.Generator, E: int, k: int):
    if cfg.routing == "single":
        return torch.zeros(T, 1, dtype=torch.int32), torch.ones(T, 1, dtype=torch.float32)
    if cfg.routing in ("softmax", "sigmoid"):
        logits = torch.randn(T, E, generator=g, dtype=torch.float32)
        scores = torch.softmax(logits, dim=-1) if cfg.routing == "softmax" else torch.sigmoid(logits)
        w, ids = torch.topk(scores, k, dim=-1, largest=True, sorted=True)
        return ids.to(torch.int32).contiguous(), _renorm(w)
    if cfg.routing == "zipf":
        p = zipf_popularity(E, cfg.zipf_s, cfg.zipf_zero_tail)
        u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_(1e-300, 1.0 - 1e-16)
        gumbel = -torch.log(-torch.log(u))
        key = torch.log(p).unsqueeze(0) + gumbel        # Gumbel-top-k: sampling without replacement ~ p
        _, ids = torch.topk(key, k, dim=-1, largest=True, sorted=True)
        z = torch.randn(T, k, generator=g, dtype=torch.float32)
        return ids.to(torch.int32).contiguous(), _renorm(torch.sigmoid(z))
    raise ValueError(cfg.routing)


def batch(cfg: MoeConfig, warmup: bool = False):
    """(x bf16 [T, H], topk_ids int32 [T, k], topk_weights fp32 [T, k]) on the CPU."""
    if warmup:
        x = activations(cfg.warmup_T, cfg.H, SEED_X_WARMUP, cfg.outliers)
        ids, w = routing(cfg, cfg.warmup_T, SEED_ROUTER_WARMUP)
    else:
        x = activations(cfg.T, cfg.H, SEED_X, cfg.outliers)
        ids, w = routing(cfg, cfg.T, SEED_ROUTER)
    return x, ids, w


def expert_w13(cfg: MoeConfig, e: int, device="cpu") -> torch.Tensor:
    """Stacked gate_up weight of expert e: [2I, H] bf16, gate rows first."""
    g = _gen(SEED_W13 + e, device)
    return (torch.randn(2 * cfg.I, cfg.H, generator=g, device=device, dtype=torch.float32) * WEIGHT_STD).to(torch.bfloat16)


def expert_w2(cfg: MoeConfig, e: int, device="cpu") -> torch.Tensor:
    """Down weight of expert e: [H, I] bf16."""
    g = _gen(SEED_W2 + e, device)
    return (torch.randn(cfg.H, cfg.I, generator=g, device=device, dtype=torch.float32) * WEIGHT_STD).to(torch.bfloat16)


def gemm_operands(cfg: GemmConfig, index: int, device="cpu"):
    """(activation bf16 [M, K] ~ N(0,1), weight bf16 [N, K] ~ N(0, 0.02))."""
    a = torch.randn(cfg.M, cfg.K, generator=_gen(SEED_X + 10 * index), dtype=torch.float32).to(torch.bfloat16)
    g = _gen(SEED_MLA + index, device)
    w = (torch.randn(cfg.N, cfg.K, generator=g, device=device, dtype=torch.float32) * WEIGHT_STD).to(torch.bfloat16)
    return a, w


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (what the oracle takes)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def router_logits(cfg: MoeConfig, device="cpu") -> torch.Tensor:
    """Router logits [T, E] fp32 ~ N(0, 1), the input of the top-k router."""
    return torch.randn(cfg.T, cfg.E, generator=_gen(SEED_LOGITS, device), device=device, dtype=torch.float32)
