"""The expert-parallel forward on this GPU with the library's experts
(LibraryExperts, library_amax) over a one-rank NCCL group: with every expert
local it must give exactly the single-device forward's output."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from nvfp4_moe_expert_topk_b200 import nvfp4_moe_forward
from nvfp4_moe_expert_topk_b200 import workloads as W
from nvfp4_moe_expert_topk_b200.ep import ExpertParallelMoE, LibraryExperts, library_amax, library_quantize
from test_gpu_moe import Problem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,dispatch", [("tiny", "bf16"), ("tiny_shared", "bf16"), ("tiny", "nvfp4"),
                                           ("tiny_shared", "nvfp4")])
def test_expert_parallel_single_rank_matches_forward(name, dispatch):
    """tiny_shared: 8 routed experts plus a shared one (slot 2, id 8, weight 1),
    served on the token's own rank as local expert 8.  nvfp4: the rows travel
    as NVFP4 codes and row-major scales (library_quantize) and the experts run
    nvfp4_moe_forward_quantized on them."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        cfg = W.MOE_CONFIGS[name]
        p = Problem(cfg)
        inputs = p.device_inputs()
        ref = torch.empty(p.x.shape[0], cfg.H, dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros_like(p.run(inputs)[1])
        nvfp4_moe_forward(**dict(inputs, x_gs=None), out=ref, workspace=ws)
        inter_gs = inputs["inter_gs"]
        ep = ExpertParallelMoE(cfg.E - cfg.shared, amax_fn=library_amax,
                               experts_fn=LibraryExperts(p.dw, inter_gs, cfg.k), num_shared=cfg.shared,
                               quantize_fn=library_quantize if dispatch == "nvfp4" else None)
        out = ep.forward(inputs["x"], inputs["topk_ids"], inputs["topk_weights"])
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
