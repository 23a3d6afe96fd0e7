"""Test-side helpers: the scale-layout definition written out in numpy (from
the layout's statement in include/nvfp4moe.h, independent of the CUDA
kernels), parity metrics, and oracle-side preparation of synthetic MoE
problems."""
import numpy as np
import torch

import oracle as O
from nvfp4_moe_expert_topk_b200 import workloads as W


def to_mma_layout(sc: np.ndarray) -> np.ndarray:
    """Row-major scales [rows, cols/16] -> bytes of the tensor-core layout:
    atom (r // 128, kb) of 512 bytes; byte (r % 32)*16 + ((r % 128)//32)*4 + j
    holds the scale of row r, 16-column block 4*kb + j; pad rows are 0."""
    rows, nblk = sc.shape
    kbs = nblk // 4
    rb = (rows + 127) // 128
    out = np.zeros(rb * kbs * 512, np.uint8)
    r = np.arange(rows)
    base = ((r // 128)[:, None] * kbs + np.arange(kbs)[None, :]) * 512 + ((r % 32) * 16 + ((r % 128) // 32) * 4)[:, None]
    for j in range(4):
        out[base + j] = sc[:, j::4]
    return out


def from_mma_layout(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    kbs = cols // 64
    r = np.arange(rows)
    base = ((r // 128)[:, None] * kbs + np.arange(kbs)[None, :]) * 512 + ((r % 32) * 16 + ((r % 128) // 32) * 4)[:, None]
    sc = np.zeros((rows, cols // 16), np.uint8)
    for j in range(4):
        sc[:, j::4] = buf[base + j]
    return sc


def from_rowblock_layout(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Scales in row blocks -> row-major [rows, cols/16]: for each 128-row
    block and 256-column k-tile, 2 KB holding 16 bytes per row, the row's
    scale of 16-column block j at (row % 128) * 16 + j % 16 of k-tile j // 16
    (the layout stated for workspace region 1 in include/nvfp4moe.h)."""
    nkt = (cols + 255) // 256
    r = np.arange(rows)[:, None]
    j = np.arange(cols // 16)[None, :]
    return buf[((r // 128) * nkt + j // 16) * 2048 + (r % 128) * 16 + j % 16]


def row_rel_l2(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    gpu = gpu.astype(np.float64)
    ref = ref.astype(np.float64)
    num = np.linalg.norm(gpu - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def row_max_rel(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """max_i |gpu - ref| / ||ref||_2 per row (the looser reading of the bar)."""
    gpu = gpu.astype(np.float64)
    ref = ref.astype(np.float64)
    den = np.linalg.norm(ref, axis=1)
    return np.abs(gpu - ref).max(axis=1) / np.where(den > 0, den, 1)


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


class OracleWeights:
    """Oracle-side NVFP4 weights (row-major scales) of selected experts,
    quantised on the CPU from the same bf16 values the device used."""

    def __init__(self, cfg, experts, device):
        self.cfg = cfg
        self.experts = list(experts)
        H, I = cfg.H, cfg.I
        n = len(self.experts)
        self.w13_codes = np.empty((n, 2 * I, H // 2), np.uint8)
        self.w13_scales = np.empty((n, 2 * I, H // 16), np.uint8)
        self.w13_gs = np.empty((n, 2), np.float32)
        self.w2_codes = np.empty((n, H, I // 2), np.uint8)
        self.w2_scales = np.empty((n, H, I // 16), np.uint8)
        self.w2_gs = np.empty(n, np.float32)
        for i, e in enumerate(self.experts):
            w13 = W.bf16_bits(W.expert_w13(cfg, e, device))
            w2 = W.bf16_bits(W.expert_w2(cfg, e, device))
            for h in range(2):
                part = w13[h * I:(h + 1) * I]
                gs = O.global_scale_bf16(part)
                c, s = O.quantize_bf16(part, gs)
                self.w13_codes[i, h * I:(h + 1) * I] = c
                self.w13_scales[i, h * I:(h + 1) * I] = s
                self.w13_gs[i, h] = gs
            gs = O.global_scale_bf16(w2)
            c, s = O.quantize_bf16(w2, gs)
            self.w2_codes[i], self.w2_scales[i], self.w2_gs[i] = c, s, gs

    def oracle_kwargs(self):
        return dict(w13_codes=self.w13_codes, w13_scales=self.w13_scales, w13_gs=self.w13_gs,
                    w2_codes=self.w2_codes, w2_scales=self.w2_scales, w2_gs=self.w2_gs)

    def remap_ids(self, ids: np.ndarray) -> np.ndarray:
        """Expert ids -> positions in self.experts (ids outside the set -> -1)."""
        lut = -np.ones(max(self.experts) + 2 if self.experts else 1, np.int64)
        lut[np.array(self.experts)] = np.arange(len(self.experts))
        out = np.where((ids >= 0) & (ids < lut.size - 1), lut[np.clip(ids, 0, lut.size - 2)], -1)
        return out.astype(np.int32)
