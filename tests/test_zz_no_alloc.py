"""nvfp4_moe_forward_noalloc: the entry point for callers that cannot allocate
device memory (a plug-in whose host framework owns all device memory, a
serving loop that cannot take cudaMalloc's device-wide synchronisation, a
deployment with a memory budget fixed at start-up).  Its scratch is one
static device array that keeps the previous call's contents, so each call
must give exactly the output of nvfp4_moe_forward with a caller workspace:
the same kernels on the same inputs, bit for bit, call after call, also when
a larger batch is followed by a smaller one (stale routing tables left in the
array must not leak into the next call).

This file is named so that pytest collects it last; it also runs on its own
in a fresh process."""
import ctypes

import pytest
import torch

from nvfp4_moe_expert_topk_b200 import (_moe_args, lib, nvfp4_global_scale,
                                        nvfp4_moe_calibrate, nvfp4_moe_forward)
from nvfp4_moe_expert_topk_b200 import prep
from nvfp4_moe_expert_topk_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
NVFP4_ERR_WORKSPACE_TOO_SMALL = -4


def _batch(cfg, T, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, cfg.H, generator=g).to(torch.bfloat16)
    ids = torch.stack([torch.randperm(cfg.E, generator=g)[:cfg.k] for _ in range(T)]).to(torch.int32)
    w = torch.rand(T, cfg.k, generator=g) + 0.1
    return x, ids, (w / w.sum(-1, keepdim=True)).float()


def test_noalloc_equals_workspace_forward_call_after_call():
    cfg = W.MOE_CONFIGS["tiny"]
    wts = prep.MoeWeights.synthetic(cfg, DEV)
    xw, idw, ww = W.batch(cfg, warmup=True)
    gsw = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(xw.to(DEV), gsw)
    inter_gs = torch.empty(cfg.E, dtype=torch.float32, device=DEV)
    nvfp4_moe_calibrate(xw.to(DEV), idw.to(DEV), ww.to(DEV), gsw, **wts.args(), inter_gs_out=inter_gs,
                        workspace=prep.workspace(cfg.warmup_T, cfg.k, cfg.E, cfg.H, cfg.I, DEV))
    stream = torch.cuda.current_stream()
    # two calls of the same shape, then a larger batch followed by a smaller one
    for call, T in enumerate([cfg.T, cfg.T, 4 * cfg.T, 24]):
        x, ids, w = _batch(cfg, T, 1000 + call)
        x, ids, w = x.to(DEV), ids.to(DEV), w.to(DEV)
        x_gs = torch.empty(1, dtype=torch.float32, device=DEV)
        nvfp4_global_scale(x, x_gs)
        ref = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=DEV)
        ws = prep.workspace(T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
        nvfp4_moe_forward(x, ids, w, x_gs, **wts.args(), inter_gs=inter_gs, out=ref, workspace=ws)
        out = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
        args = _moe_args(x, ids, w, x_gs, **wts.args(), inter_gs=inter_gs, out=out)
        status = lib().nvfp4_moe_forward_noalloc(ctypes.byref(args), ctypes.c_void_p(stream.cuda_stream))
        assert status == 0, status
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert torch.equal(out, ref), (call, T)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = W.MOE_CONFIGS["tiny"]
    wts = prep.MoeWeights.synthetic(cfg, DEV)
    x = torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    ids = torch.zeros(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.ones(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    gs = torch.ones(1, dtype=torch.float32, device=DEV)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    args = _moe_args(x, ids, w, gs, **wts.args(), inter_gs=torch.ones(cfg.E, device=DEV), out=out)
    args.T, args.H, args.I, args.E, args.k = 4096, 7168, 3072, 384, 6      # ~1 GB of scratch needed
    status = lib().nvfp4_moe_forward_noalloc(ctypes.byref(args), None)
    assert status == NVFP4_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
