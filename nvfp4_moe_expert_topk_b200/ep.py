"""Expert parallelism (EP) of the routed-expert MoE block over a process group.

The pages' deployment splits the 384 experts over 8 ranks, 48 per rank
("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 1 "Config values"; page 3
"Architecture Notes").  Rank r owns experts [r*El, (r+1)*El), El = E / W,
and holds its own batch of tokens.  One forward:

  1. global scale: every rank reduces max|x| over its batch, the maximum over
     the ranks is taken (one all-reduce of one float), gs = 2688 / amax (1 if
     amax = 0): the scale one device would compute for the union batch;
  2. dispatch: each token goes once to every rank that owns one of its top-k
     experts, with its k ids rewritten to that rank's local ids (-1 for the
     slots whose expert lives elsewhere: the forward's skipped-slot rule) and
     its k weights; row counts are exchanged first, then the rows, ids and
     weights with uneven all-to-alls.  With a quantize_fn the rows travel as
     NVFP4: each rank quantises its batch once with the global scale of step
     1 and sends codes and row-major scales (H/2 + H/16 bytes a row, 4032 at
     H = 7168, against 14336 for bf16); the receiving rank's forward only
     permutes them (nvfp4_moe_forward_quantized), so the result is the one
     of bf16 dispatch bit for bit;
  3. each rank runs the MoE block on the rows it received with its own
     experts: the weighted sum over the token's local slots;
  4. combine: the partial outputs go back to the token's rank (all-to-all
     again) and are summed there in fp32 in ascending rank order, then stored
     in x's dtype.

Shared experts (the routed chain with one expert and no routing, page 1
"Phase 1") are replicated on every rank.  Their slots arrive the way the
router with shared experts writes them: ids E .. E + num_shared - 1 (weight 1).
A token's shared slots are served on its own rank, as local experts
El .. El + num_shared - 1 after the rank's routed ones, so the shared experts
run as extra groups of the rank's local forward and add no traffic.

The counts exchange reads the counts on the host, so a forward synchronises
once with the device.  The per-rank compute is a pluggable callable; on a GPU
it is the library's nvfp4_moe_forward (`LibraryExperts`).
"""
from typing import Callable, Optional

import numpy as np
import torch
import torch.distributed as dist

GS_NUMERATOR = np.float32(2688.0)   # 448 * 6: largest E4M3 scale times largest E2M1 value


def global_scale_from_amax(amax: float) -> np.float32:
    """2688 / amax rounded to fp32 (IEEE division), 1 when amax is 0."""
    a = np.float32(amax)
    return np.float32(1.0) if a == 0 else np.float32(GS_NUMERATOR / a)


class ExpertParallelMoE:
    """One rank's side of an expert-parallel MoE forward.

    amax_fn(x) -> float: max|x| of the local batch.
    experts_fn(x_recv, local_ids, weights, gs) -> [n, H]: the MoE block of
    this rank's experts on received rows (local_ids < 0 are skipped slots;
    El .. El + num_shared - 1 are the shared experts); x_recv is a bf16
    [n, H] tensor, or with a quantize_fn the pair (codes [n, H/2], scales
    [n, H/16]) of NVFP4 rows made with global scale gs.
    quantize_fn(x, gs) -> (codes, scales): NVFP4 quantisation of the local
    batch with a given global scale (None: dispatch bf16 rows).
    num_experts counts the routed experts only."""

    def __init__(self, num_experts: int, amax_fn: Callable, experts_fn: Callable,
                 group: Optional[dist.ProcessGroup] = None, num_shared: int = 0,
                 quantize_fn: Optional[Callable] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if num_experts % self.world != 0:
            raise ValueError(f"{num_experts} experts do not split evenly over {self.world} ranks")
        self.E = num_experts
        self.El = num_experts // self.world
        self.first_expert = self.rank * self.El
        if num_shared < 0:
            raise ValueError("num_shared must be >= 0")
        self.num_shared = num_shared
        self.amax_fn = amax_fn
        self.experts_fn = experts_fn
        self.quantize_fn = quantize_fn

    # ------------------------------------------------------------ steps
    def batch_global_scale(self, x: torch.Tensor) -> np.float32:
        a = float(self.amax_fn(x)) if x.numel() else 0.0     # a rank without tokens adds nothing
        t = torch.tensor([a], dtype=torch.float32, device=x.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)
        return global_scale_from_amax(t.item())

    def plan(self, topk_ids: torch.Tensor):
        """For each destination rank d: the tokens with a slot on d (ascending)
        and their ids rewritten to d's local expert ids (-1 elsewhere).
        Shared-expert slots (id >= E) stay on this rank, as local ids
        El + (id - E)."""
        ids = topk_ids.to(torch.int64)
        shared = ids >= self.E
        dest = torch.where(ids >= 0, ids // self.El, torch.full_like(ids, -1))
        dest = torch.where(shared, torch.full_like(ids, self.rank), dest)
        local_all = torch.where(shared, ids - self.E + self.El, ids - dest * self.El)
        tokens, local_ids = [], []
        for d in range(self.world):
            on_d = dest == d
            sel = torch.nonzero(on_d.any(dim=1), as_tuple=False).flatten()
            tokens.append(sel)
            local_ids.append(torch.where(on_d[sel], local_all[sel], torch.full_like(ids[sel], -1)).to(torch.int32))
        return tokens, local_ids

    def _exchange(self, send: torch.Tensor, send_counts, recv_counts) -> torch.Tensor:
        recv = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(recv, send.contiguous(), list(recv_counts), list(send_counts), group=self.group)
        return recv

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
        """out [T, H] in out_dtype (default x.dtype) for this rank's tokens."""
        T, H = x.shape
        if topk_ids.numel() and int(topk_ids.max()) >= self.E + self.num_shared:
            raise ValueError(f"expert id >= {self.E + self.num_shared} (routed + shared experts)")
        gs = self.batch_global_scale(x)
        tokens, local_ids = self.plan(topk_ids)
        send_counts = [int(t.numel()) for t in tokens]
        c = torch.tensor(send_counts, dtype=torch.int64, device=x.device)
        rc = torch.empty_like(c)
        dist.all_to_all_single(rc, c, group=self.group)
        recv_counts = [int(v) for v in rc.tolist()]
        order = torch.cat(tokens)
        if self.quantize_fn is None:
            recv_x = self._exchange(x[order], send_counts, recv_counts)
        else:
            codes, scales = self.quantize_fn(x, gs)
            recv_x = (self._exchange(codes[order], send_counts, recv_counts),
                      self._exchange(scales[order], send_counts, recv_counts))
        recv_ids = self._exchange(torch.cat(local_ids), send_counts, recv_counts)
        recv_w = self._exchange(topk_weights[order].to(torch.float32), send_counts, recv_counts)
        y = self.experts_fn(recv_x, recv_ids, recv_w, gs)
        back = self._exchange(y, recv_counts, send_counts)
        out = torch.zeros((T, H), dtype=torch.float32, device=x.device)
        start = 0
        for d in range(self.world):            # fixed order: deterministic sums
            n = send_counts[d]
            if n:
                out.index_add_(0, tokens[d], back[start:start + n].to(torch.float32))
            start += n
        return out.to(out_dtype or x.dtype)


class LibraryExperts:
    """experts_fn backed by the library on this rank's GPU: nvfp4_moe_forward
    over the local experts' NVFP4 weights (a prep.MoeWeights of El experts,
    then the shared experts) and their warmup inter_gs; the workspace grows
    with the received rows."""

    def __init__(self, weights, inter_gs: torch.Tensor, top_k: int):
        self.weights = weights
        self.inter_gs = inter_gs
        self.k = top_k
        self.ws = None

    def __call__(self, x, local_ids, weights, gs):
        from . import nvfp4_moe_forward, nvfp4_moe_forward_quantized, nvfp4_moe_workspace_size
        w = self.weights
        quantised = isinstance(x, tuple)
        dev = x[0].device if quantised else x.device
        n = x[0].shape[0] if quantised else x.shape[0]
        out = torch.empty((n, w.H), dtype=torch.bfloat16, device=dev)
        if n == 0:
            return out
        need = nvfp4_moe_workspace_size(n, self.k, w.E, w.H, w.I)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        x_gs = torch.tensor([float(gs)], dtype=torch.float32, device=dev)
        if quantised:
            nvfp4_moe_forward_quantized(x[0].contiguous(), x[1].contiguous(), local_ids.contiguous(),
                                        weights.contiguous(), x_gs, **w.args(), inter_gs=self.inter_gs, out=out,
                                        workspace=self.ws)
        else:
            nvfp4_moe_forward(x.contiguous(), local_ids.contiguous(), weights.contiguous(), x_gs, **w.args(),
                              inter_gs=self.inter_gs, out=out, workspace=self.ws)
        return out


def library_amax(x: torch.Tensor) -> float:
    """amax_fn backed by the library (nvfp4_amax) for bf16 CUDA tensors."""
    from . import nvfp4_amax
    a = torch.empty(1, dtype=torch.float32, device=x.device)
    nvfp4_amax(x.contiguous(), a)
    return a.item()


def library_quantize(x: torch.Tensor, gs) -> tuple:
    """quantize_fn backed by the library (nvfp4_quantize, row-major scales):
    codes uint8 [T, H/2] and scales uint8 [T, H/16] of a bf16 CUDA tensor
    with the given global scale."""
    from . import NVFP4_SCALES_ROWMAJOR, nvfp4_quantize
    T, H = x.shape
    codes = torch.empty((T, H // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((T, H // 16), dtype=torch.uint8, device=x.device)
    if T:
        g = torch.tensor([float(gs)], dtype=torch.float32, device=x.device)
        nvfp4_quantize(x.contiguous(), g, codes, scales, NVFP4_SCALES_ROWMAJOR)
    return codes, scales
