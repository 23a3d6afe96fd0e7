"""nvfp4_moe_forward_noalloc: the entry point for callers that cannot allocate
device memory (graph-capture code, plug-ins whose host owns all device
memory, paths that cannot take cudaMalloc's synchronisation).  It must give
the same output as nvfp4_moe_forward with a caller workspace, call after
call, while the scratch array keeps the previous call's contents.

This file is named so that pytest collects it last; it also runs on its own
in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from helpers import bf16_to_np, cosine, row_rel_l2
from nvfp4_moe_expert_topk_b200 import (_moe_args, lib, nvfp4_global_scale,
                                        nvfp4_moe_calibrate, nvfp4_moe_forward)
from nvfp4_moe_expert_topk_b200 import prep
from nvfp4_moe_expert_topk_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROW_TOL = 2e-2          # the output bar of the MoE parity tests
COS_TOL = 0.9995
NVFP4_ERR_WORKSPACE_TOO_SMALL = -4


def _batch(cfg, call):
    if call == 0:
        return W.batch(cfg)
    g = torch.Generator().manual_seed(1000 + call)
    x = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16)
    ids = torch.stack([torch.randperm(cfg.E, generator=g)[:cfg.k] for _ in range(cfg.T)]).to(torch.int32)
    w = torch.rand(cfg.T, cfg.k, generator=g) + 0.1
    return x, ids, (w / w.sum(-1, keepdim=True)).float()


def test_noalloc_matches_workspace_forward_two_calls():
    cfg = W.MOE_CONFIGS["tiny"]
    wts = prep.MoeWeights.synthetic(cfg, DEV)
    xw, idw, ww = W.batch(cfg, warmup=True)
    gsw = torch.empty(1, dtype=torch.float32, device=DEV)
    nvfp4_global_scale(xw.to(DEV), gsw)
    inter_gs = torch.empty(cfg.E, dtype=torch.float32, device=DEV)
    nvfp4_moe_calibrate(xw.to(DEV), idw.to(DEV), ww.to(DEV), gsw, **wts.args(), inter_gs_out=inter_gs,
                        workspace=prep.workspace(cfg.warmup_T, cfg.k, cfg.E, cfg.H, cfg.I, DEV))
    ws = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, DEV)
    stream = torch.cuda.current_stream()
    for call in range(2):
        x, ids, w = _batch(cfg, call)
        x, ids, w = x.to(DEV), ids.to(DEV), w.to(DEV)
        x_gs = torch.empty(1, dtype=torch.float32, device=DEV)
        nvfp4_global_scale(x, x_gs)
        ref = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
        nvfp4_moe_forward(x, ids, w, x_gs, **wts.args(), inter_gs=inter_gs, out=ref, workspace=ws)
        out = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
        args = _moe_args(x, ids, w, x_gs, **wts.args(), inter_gs=inter_gs, out=out)
        status = lib().nvfp4_moe_forward_noalloc(ctypes.byref(args), ctypes.c_void_p(stream.cuda_stream))
        assert status == 0, status
        torch.cuda.synchronize()
        got, want = bf16_to_np(out), bf16_to_np(ref)
        assert np.all(np.isfinite(got))
        assert row_rel_l2(got, want).max() <= ROW_TOL
        assert cosine(got, want) >= COS_TOL


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
