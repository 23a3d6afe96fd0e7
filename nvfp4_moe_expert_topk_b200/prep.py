"""Weight and buffer preparation through the library's own entry points.

Quantising a bf16 weight is: nvfp4_global_scale (gs = 2688 / amax) followed
by nvfp4_quantize into codes [rows, cols/2] and scales in the tensor-core
layout.  The stacked gate_up weight of an expert gets one global scale per
half ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 1 "Phase 2": dual global
scales, same pattern as the MoE gate+up).
"""
import torch

from . import (NVFP4_SCALES_MMA, nvfp4_global_scale, nvfp4_moe_workspace_size, nvfp4_quantize,
               nvfp4_scales_bytes)
from . import workloads as W


def quantize(x, gs=None, scale_layout=NVFP4_SCALES_MMA, stream=None):
    """bf16 [rows, cols] CUDA tensor -> (codes, scales, gs [1]); gs computed from x if not given."""
    rows, cols = x.shape
    if gs is None:
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
        nvfp4_global_scale(x, gs, stream)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(nvfp4_scales_bytes(rows, cols, scale_layout), dtype=torch.uint8, device=x.device)
    nvfp4_quantize(x, gs, codes, scales, scale_layout, stream)
    return codes, scales, gs


class MoeWeights:
    """NVFP4 weights of E experts on one device:
    w13_codes [E, 2I, H/2], w13_scales (MMA layout of [E*2I, H]), w13_gs [E, 2],
    w2_codes [E, H, I/2], w2_scales (MMA layout of [E*H, I]), w2_gs [E]."""

    def __init__(self, E, H, I, device):
        self.E, self.H, self.I = E, H, I
        self.w13_codes = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=device)
        self.w13_scales = torch.empty(E * 2 * I * (H // 16), dtype=torch.uint8, device=device)
        self.w13_gs = torch.empty(E, 2, dtype=torch.float32, device=device)
        self.w2_codes = torch.empty(E, H, I // 2, dtype=torch.uint8, device=device)
        self.w2_scales = torch.empty(E * H * (I // 16), dtype=torch.uint8, device=device)
        self.w2_gs = torch.empty(E, dtype=torch.float32, device=device)

    def set_expert(self, e, w13, w2, stream=None):
        """Quantise expert e from bf16 w13 [2I, H] (gate rows first) and w2 [H, I]."""
        H, I = self.H, self.I
        s13 = 2 * I * (H // 16)
        s2 = H * (I // 16)
        half = I * (H // 16)
        for h in range(2):
            src = w13[h * I:(h + 1) * I]
            gs = self.w13_gs[e, h:h + 1]
            nvfp4_global_scale(src, gs, stream)
            nvfp4_quantize(src, gs, self.w13_codes[e, h * I:(h + 1) * I],
                           self.w13_scales[e * s13 + h * half:e * s13 + (h + 1) * half], NVFP4_SCALES_MMA, stream)
        nvfp4_global_scale(w2, self.w2_gs[e:e + 1], stream)
        nvfp4_quantize(w2, self.w2_gs[e:e + 1], self.w2_codes[e], self.w2_scales[e * s2:(e + 1) * s2],
                       NVFP4_SCALES_MMA, stream)

    @classmethod
    def synthetic(cls, cfg, device):
        """Seeded N(0, 0.02) weights of a workload config, quantised on the device."""
        wts = cls(cfg.E, cfg.H, cfg.I, device)
        for e in range(cfg.E):
            wts.set_expert(e, W.expert_w13(cfg, e, device), W.expert_w2(cfg, e, device))
        return wts

    def args(self):
        return dict(w13_codes=self.w13_codes, w13_scales=self.w13_scales, w13_gs=self.w13_gs,
                    w2_codes=self.w2_codes, w2_scales=self.w2_scales, w2_gs=self.w2_gs)


def workspace(T, k, E, H, I, device):
    """Zeroed workspace for nvfp4_moe_forward / nvfp4_moe_calibrate."""
    n = nvfp4_moe_workspace_size(T, k, E, H, I)
    if n == 0:
        raise ValueError("unsupported MoE shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)
