"""The C-ABI library builds, loads and exports every entry point of
include/nvfp4moe.h; host-only entry points and argument checks work without a
GPU (no kernel is launched here)."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "nvfp4moe.h")


@pytest.fixture(scope="module")
def L():
    from nvfp4_moe_expert_topk_b200 import build, lib
    build.build()
    return lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\s*\*?\s*(nvfp4_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["nvfp4_quantize", "nvfp4_gemm", "nvfp4_moe_forward", "nvfp4_global_scale",
                 "nvfp4_swizzle_scales", "nvfp4_moe_workspace_size", "nvfp4_moe_get_error",
                 "nvfp4_moe_route_debug", "nvfp4_moe_calibrate", "nvfp4_status_string", "nvfp4_moe_topk", "nvfp4_moe_topk_shared",
                 "nvfp4_moe_forward_noalloc", "nvfp4_moe_forward_timed", "nvfp4_moe_forward_quantized"]:
        assert want in names


def test_library_exports_every_declared_symbol(L):
    from nvfp4_moe_expert_topk_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_status_strings(L):
    from nvfp4_moe_expert_topk_b200 import nvfp4_status_string
    assert nvfp4_status_string(0) == "NVFP4_OK"
    for code in range(-1, -9, -1):
        assert nvfp4_status_string(code).startswith("NVFP4_ERR_")
    assert nvfp4_status_string(-99) == "NVFP4_ERR_UNKNOWN"


def test_sizes_host_only(L):
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_workspace_region, nvfp4_moe_workspace_size, nvfp4_scales_bytes
    assert nvfp4_scales_bytes(100, 256, 0) == 100 * 16
    assert nvfp4_scales_bytes(100, 256, 1) == 128 * 16
    assert nvfp4_scales_bytes(100, 48, 1) == -1
    assert nvfp4_scales_bytes(100, 40, 0) == -1
    ws = nvfp4_moe_workspace_size(4096, 6, 384, 7168, 3072)
    R = 4096 * 6
    mt_max = (R + 127 * 384) // 128
    assert ws >= mt_max * 128 * (7168 // 2 + 7168 // 16 + 3072 // 2 + 3072 // 16) + R * 7168 * 2
    assert nvfp4_moe_workspace_size(64, 6, 48, 7168, 3000) == 0          # I % 128 != 0
    assert nvfp4_moe_workspace_size(64, 33, 48, 7168, 3072) == 0         # k > 32
    assert nvfp4_moe_workspace_size(0, 6, 48, 7168, 3072) > 0
    off, n = nvfp4_moe_workspace_region(64, 6, 48, 7168, 3072, 4)
    assert off % 1024 == 0 and n == 64 * 6 * 7168 * 2
    end = 0
    for region in range(8):
        o, n = nvfp4_moe_workspace_region(64, 6, 48, 7168, 3072, region)
        assert o + n <= nvfp4_moe_workspace_size(64, 6, 48, 7168, 3072)


def test_argument_checks_before_any_launch(L):
    P = ctypes.c_void_p
    fake = P(1 << 40)                          # never dereferenced: the checks fail first
    assert L.nvfp4_quantize(None, 4, 64, 64, fake, fake, fake, 0, None) == -1
    assert L.nvfp4_quantize(fake, 4, 40, 64, fake, fake, fake, 0, None) == -2          # cols % 16
    assert L.nvfp4_quantize(fake, 4, 48, 48, fake, fake, fake, 1, None) == -2          # MMA layout, cols % 64
    assert L.nvfp4_quantize(fake, 4, 64, 64, fake, fake, fake, 7, None) == -1          # bad layout
    assert L.nvfp4_quantize(P((1 << 40) + 4), 4, 64, 64, fake, fake, fake, 0, None) == -3
    seg = (ctypes.c_int64 * 1)(256)
    cseg = ctypes.cast(seg, P)
    assert L.nvfp4_gemm(fake, fake, fake, 8, fake, fake, fake, cseg, 1, 256, 100, fake, 256, None) == -2   # K % 64
    assert L.nvfp4_gemm(fake, fake, fake, 8, fake, fake, fake, cseg, 1, 200, 128, fake, 256, None) == -2   # N % 128
    bad = (ctypes.c_int64 * 2)(100, 256)
    assert L.nvfp4_gemm(fake, fake, fake, 8, fake, fake, fake, ctypes.cast(bad, P), 2, 256, 128, fake, 256,
                        None) == -1                                                     # segment end % 32
    assert L.nvfp4_gemm(fake, fake, fake, 8, fake, fake, fake, cseg, 1, 256, 128, fake, 100, None) == -1   # ldo < N
    assert L.nvfp4_moe_forward(None, fake, 1 << 30, None) == -1
    assert L.nvfp4_moe_forward_noalloc(None, None) == -1
    assert L.nvfp4_moe_get_error(None, None, None) == -1


def test_moe_forward_checks(L):
    from nvfp4_moe_expert_topk_b200 import MoeArgs
    a = MoeArgs()
    F = 1 << 40
    a.x = a.topk_ids = a.topk_weights = a.x_gs = a.w13_codes = a.w13_scales = F
    a.w13_gs = a.w2_codes = a.w2_scales = a.w2_gs = a.inter_gs = a.out = F
    a.T, a.H, a.I, a.E, a.k = 64, 7168, 3072, 48, 6
    assert L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1024, None) == -4     # workspace too small
    a.I = 3000
    assert L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1 << 40, None) == -2
    a.I = 3072
    a.w2_codes = F + 8
    assert L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1 << 40, None) == -3
    assert L.nvfp4_moe_forward_noalloc(ctypes.byref(a), None) == -3    # checked before the scratch is touched
    a.w2_codes = None
    assert L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1 << 40, None) == -1
    assert L.nvfp4_moe_forward_noalloc(ctypes.byref(a), None) == -1
    a.w2_codes = F
    a.out = None
    assert L.nvfp4_moe_forward_noalloc(ctypes.byref(a), None) == -1
    a.out = F
    # pre-quantised activations: x may be NULL, x_gs and both code buffers are required
    a.x = None
    a.w2_codes = None
    assert L.nvfp4_moe_forward_quantized(ctypes.byref(a), ctypes.c_void_p(F), ctypes.c_void_p(F),
                                         ctypes.c_void_p(F), 1 << 40, None) == -1     # w2_codes NULL
    a.w2_codes = F
    assert L.nvfp4_moe_forward_quantized(ctypes.byref(a), None, ctypes.c_void_p(F), ctypes.c_void_p(F),
                                         1 << 40, None) == -1
    assert L.nvfp4_moe_forward_quantized(ctypes.byref(a), ctypes.c_void_p(F + 4), ctypes.c_void_p(F),
                                         ctypes.c_void_p(F), 1 << 40, None) == -3
    a.x_gs = None
    assert L.nvfp4_moe_forward_quantized(ctypes.byref(a), ctypes.c_void_p(F), ctypes.c_void_p(F),
                                         ctypes.c_void_p(F), 1 << 40, None) == -1
    # an empty batch: its pointers may be NULL (the checks pass; without a GPU the
    # call then stops at the device check), the weights' may not
    a.T = 0
    a.x = a.topk_ids = a.topk_weights = a.x_gs = a.out = None
    no_device = L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1 << 40, None)
    assert no_device not in (-1, -2, -3, -4), no_device
    assert L.nvfp4_moe_forward_quantized(ctypes.byref(a), None, None, ctypes.c_void_p(F), 1 << 40,
                                         None) == no_device
    a.w13_codes = None
    assert L.nvfp4_moe_forward(ctypes.byref(a), ctypes.c_void_p(F), 1 << 40, None) == -1


def test_topk_checks(L):
    P = ctypes.c_void_p
    F = P(1 << 40)
    assert L.nvfp4_moe_topk(None, 4, 48, 6, 0, F, F, None) == -1
    assert L.nvfp4_moe_topk(F, -1, 48, 6, 0, F, F, None) == -1
    assert L.nvfp4_moe_topk(F, 4, 48, 0, 0, F, F, None) == -1
    assert L.nvfp4_moe_topk(F, 4, 48, 6, 2, F, F, None) == -1         # unknown scoring
    assert L.nvfp4_moe_topk(F, 4, 1025, 6, 0, F, F, None) == -2      # E > 1024
    assert L.nvfp4_moe_topk(F, 4, 48, 33, 0, F, F, None) == -2       # k > 32
    assert L.nvfp4_moe_topk(F, 4, 4, 6, 1, F, F, None) == -2         # k > E
    # the same checks with shared-expert slots, plus the slot and expert limits
    assert L.nvfp4_moe_topk_shared(None, 4, 48, 6, 0, 1, F, F, None) == -1
    assert L.nvfp4_moe_topk_shared(F, 4, 48, 6, 0, -1, F, F, None) == -1     # num_shared < 0
    assert L.nvfp4_moe_topk_shared(F, 4, 48, 6, 3, 1, F, F, None) == -1      # unknown scoring
    assert L.nvfp4_moe_topk_shared(F, 4, 48, 30, 0, 3, F, F, None) == -2     # k + num_shared > 32
    assert L.nvfp4_moe_topk_shared(F, 4, 1020, 6, 0, 5, F, F, None) == -2    # E + num_shared > 1024


def test_ceiling_checks(L):
    F = ctypes.c_void_p(1 << 40)
    assert L.nvfp4_fp4_mma_ceiling(256, 10, 148, None, None, None) == -1
    assert L.nvfp4_fp4_mma_ceiling(192, 10, 148, F, None, None) == -1
    assert L.nvfp4_fp4_mma_ceiling(256, 0, 148, F, None, None) == -1
    assert L.nvfp4_fp4_mma_ceiling(256, (1 << 24) + 1, 148, F, None, None) == -2
    # TMA streaming probe: shape and alignment checks before any device work
    assert L.nvfp4_tma_stream_ceiling(None, 256, 128, 1, 4, None, None) == -1
    assert L.nvfp4_tma_stream_ceiling(F, 128, 128, 1, 4, None, None) == -1        # rows < 256
    assert L.nvfp4_tma_stream_ceiling(F, 256, 128, 0, 4, None, None) == -1        # no work
    assert L.nvfp4_tma_stream_ceiling(F, 256, 128, 1, 1, None, None) == -1        # stages < 2
    assert L.nvfp4_tma_stream_ceiling(F, 384, 128, 1, 4, None, None) == -2        # rows % 256
    assert L.nvfp4_tma_stream_ceiling(F, 256, 192, 1, 4, None, None) == -2        # row_bytes % 128
    assert L.nvfp4_tma_stream_ceiling(F, 256, 128, 1, 7, None, None) == -2        # stages > 6
    assert L.nvfp4_tma_stream_ceiling(ctypes.c_void_p((1 << 40) + 8), 256, 128, 1, 4, None, None) == -3


def test_moe_plan(L):
    from nvfp4_moe_expert_topk_b200 import nvfp4_moe_plan
    assert nvfp4_moe_plan(64, 6, 48, 7168, 3072) == (True, 0)       # decode: fused, 1-CTA tiles
    assert nvfp4_moe_plan(4096, 6, 384, 7168, 3072) == (True, 1)    # prefill: heavy experts' pairs + fused rest
    assert nvfp4_moe_plan(512, 6, 48, 7168, 3072) == (True, 1)      # the 48-expert prefill slice
    assert nvfp4_moe_plan(256, 1, 1, 7168, 3072) == (False, 2)      # shared expert: every m-tile on pairs
    assert nvfp4_moe_plan(64, 2, 4, 384, 256) == (False, 0)         # H % 256 != 0: 128-wide L2 tiles
    import ctypes
    f = ctypes.c_int32()
    assert L.nvfp4_moe_plan(64, 6, 48, 7000, 3072, ctypes.byref(f), ctypes.byref(f)) == -2
    assert L.nvfp4_moe_plan(64, 6, 48, 7168, 3072, None, None) == -1
