"""NVFP4 (W4A4) routed-expert MoE on B200: Python binding of libnvfp4moe.so.

Argument marshalling only: every step of the chain runs in the CUDA kernels
of libnvfp4moe.so (C ABI in include/nvfp4moe.h).  Tensors are torch CUDA
tensors (PyTorch provides device memory and streams); each function passes
their device pointers and the current CUDA stream to the entry point of the
same name and raises Nvfp4Error on a non-zero status.  There is no fallback:
if the library is missing, the first call raises.
"""
import ctypes
import os

import torch

__all__ = [
    "Nvfp4Error", "lib", "NVFP4_SCALES_ROWMAJOR", "NVFP4_SCALES_MMA",
    "nvfp4_status_string", "nvfp4_global_scale", "nvfp4_scales_bytes", "nvfp4_quantize",
    "nvfp4_swizzle_scales", "nvfp4_gemm", "nvfp4_moe_workspace_size", "nvfp4_moe_forward",
    "nvfp4_moe_forward_timed", "nvfp4_moe_forward_noalloc", "nvfp4_moe_forward_quantized",
    "nvfp4_moe_calibrate", "nvfp4_moe_route_debug", "nvfp4_moe_workspace_region",
    "nvfp4_moe_get_error", "nvfp4_moe_topk", "nvfp4_moe_topk_shared", "NVFP4_SCORING_SOFTMAX",
    "NVFP4_SCORING_SIGMOID", "nvfp4_fp4_mma_ceiling", "nvfp4_tma_stream_ceiling", "nvfp4_moe_plan", "nvfp4_amax", "nvfp4_debug_bounded_wait",
    "MoeArgs",
]

NVFP4_SCALES_ROWMAJOR = 0
NVFP4_SCALES_MMA = 1
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4moe.so")

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {nvfp4_status_string(status)} ({status})")


class MoeArgs(ctypes.Structure):
    """Mirror of nvfp4_moe_args."""
    _fields_ = [
        ("x", ctypes.c_void_p), ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
        ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("topk_ids", ctypes.c_void_p), ("topk_weights", ctypes.c_void_p), ("x_gs", ctypes.c_void_p),
        ("w13_codes", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p), ("w13_gs", ctypes.c_void_p),
        ("w2_codes", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p), ("w2_gs", ctypes.c_void_p),
        ("inter_gs", ctypes.c_void_p), ("out", ctypes.c_void_p),
    ]


def lib():
    """The loaded libnvfp4moe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m nvfp4_moe_expert_topk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.nvfp4_status_string.argtypes = [i32]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_global_scale.argtypes = [P, i64, P, P]
        L.nvfp4_scales_bytes.argtypes = [i64, i64, i32]
        L.nvfp4_scales_bytes.restype = i64
        L.nvfp4_quantize.argtypes = [P, i64, i64, i64, P, P, P, i32, P]
        L.nvfp4_swizzle_scales.argtypes = [P, i64, i64, i64, P, P]
        L.nvfp4_gemm.argtypes = [P, P, P, i64, P, P, P, P, i32, i64, i64, P, i64, P]
        L.nvfp4_moe_workspace_size.argtypes = [i64, i32, i32, i64, i64]
        L.nvfp4_moe_workspace_size.restype = ctypes.c_size_t
        L.nvfp4_moe_forward.argtypes = [ctypes.POINTER(MoeArgs), P, ctypes.c_size_t, P]
        L.nvfp4_moe_forward_timed.argtypes = [ctypes.POINTER(MoeArgs), P, ctypes.c_size_t, P,
                                              ctypes.POINTER(ctypes.c_void_p)]
        L.nvfp4_moe_forward_noalloc.argtypes = [ctypes.POINTER(MoeArgs), P]
        L.nvfp4_moe_forward_quantized.argtypes = [ctypes.POINTER(MoeArgs), P, P, P, ctypes.c_size_t, P]
        L.nvfp4_moe_calibrate.argtypes = [ctypes.POINTER(MoeArgs), P, P, ctypes.c_size_t, P]
        L.nvfp4_moe_route_debug.argtypes = [P, i64, i32, i32, P, P, P, P, ctypes.c_size_t, P]
        L.nvfp4_moe_workspace_region.argtypes = [i64, i32, i32, i64, i64, i32,
                                                 ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.nvfp4_moe_get_error.argtypes = [P, ctypes.POINTER(ctypes.c_int32), P]
        L.nvfp4_moe_topk.argtypes = [P, i64, i32, i32, i32, P, P, P]
        L.nvfp4_moe_topk_shared.argtypes = [P, i64, i32, i32, i32, i32, P, P, P]
        L.nvfp4_amax.argtypes = [P, i64, P, P]
        L.nvfp4_debug_bounded_wait.argtypes = [P, i32, P, P]
        L.nvfp4_fp4_mma_ceiling.argtypes = [i32, i32, i32, P, P, P]
        L.nvfp4_tma_stream_ceiling.argtypes = [P, i64, i64, i64, i32, P, P]
        L.nvfp4_moe_plan.argtypes = [i64, i32, i32, i64, i64, ctypes.POINTER(ctypes.c_int32),
                                     ctypes.POINTER(ctypes.c_int32)]
        _lib = L
    return _lib


def nvfp4_status_string(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()


def _check(status, where):
    if status != 0:
        raise Nvfp4Error(status, where)


def _dev(t, name, dtype=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def nvfp4_global_scale(x, gs_out, stream=None):
    """gs_out (float32 [1]) = 2688 / max|x| for a bf16 tensor x."""
    _check(lib().nvfp4_global_scale(_dev(x, "x", torch.bfloat16), x.numel(), _dev(gs_out, "gs_out", torch.float32),
                                    _stream(stream)), "nvfp4_global_scale")


def nvfp4_scales_bytes(rows, cols, scale_layout):
    return int(lib().nvfp4_scales_bytes(rows, cols, scale_layout))


def nvfp4_quantize(x, gs, codes, scales, scale_layout=NVFP4_SCALES_MMA, stream=None):
    """x bf16 [rows, cols] -> codes uint8 [rows, cols/2] and scales (uint8, layout per scale_layout)."""
    rows, cols = x.shape
    _check(lib().nvfp4_quantize(_dev(x, "x", torch.bfloat16), rows, cols, cols, _dev(gs, "gs", torch.float32),
                                _dev(codes, "codes", torch.uint8), _dev(scales, "scales", torch.uint8),
                                scale_layout, _stream(stream)), "nvfp4_quantize")


def nvfp4_swizzle_scales(inp, out, batch, rows, cols, stream=None):
    _check(lib().nvfp4_swizzle_scales(_dev(inp, "in", torch.uint8), batch, rows, cols,
                                      _dev(out, "out", torch.uint8), _stream(stream)), "nvfp4_swizzle_scales")


def nvfp4_gemm(a_codes, a_scales, a_gs, b_codes, b_scales, b_gs, seg_end, out, stream=None):
    """out bf16 [M, N] = A [M, K] x B [N, K]^T in NVFP4 (scales in the MMA layout)."""
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    seg = (ctypes.c_int64 * len(seg_end))(*[int(v) for v in seg_end])
    _check(lib().nvfp4_gemm(_dev(a_codes, "a_codes", torch.uint8), _dev(a_scales, "a_scales", torch.uint8),
                            _dev(a_gs, "a_gs", torch.float32), M, _dev(b_codes, "b_codes", torch.uint8),
                            _dev(b_scales, "b_scales", torch.uint8), _dev(b_gs, "b_gs", torch.float32),
                            ctypes.cast(seg, ctypes.c_void_p), len(seg_end), N, K,
                            _dev(out, "out", torch.bfloat16), out.stride(0), _stream(stream)), "nvfp4_gemm")


def nvfp4_moe_workspace_size(T, k, E, H, I):
    return int(lib().nvfp4_moe_workspace_size(T, k, E, H, I))


def _moe_args(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
              inter_gs, out, x_shape=None):
    T, H = x.shape if x is not None else x_shape
    E, twoI = w13_codes.shape[0], w13_codes.shape[1]
    a = MoeArgs()
    a.x = None if x is None else _dev(x, "x", torch.bfloat16).value
    a.T, a.H, a.I, a.E, a.k = T, H, twoI // 2, E, topk_ids.shape[1]
    a.topk_ids = _dev(topk_ids, "topk_ids", torch.int32).value
    a.topk_weights = _dev(topk_weights, "topk_weights", torch.float32).value
    a.x_gs = None if x_gs is None else _dev(x_gs, "x_gs", torch.float32).value   # None: from this batch
    a.w13_codes = _dev(w13_codes, "w13_codes", torch.uint8).value
    a.w13_scales = _dev(w13_scales, "w13_scales", torch.uint8).value
    a.w13_gs = _dev(w13_gs, "w13_gs", torch.float32).value
    a.w2_codes = _dev(w2_codes, "w2_codes", torch.uint8).value
    a.w2_scales = _dev(w2_scales, "w2_scales", torch.uint8).value
    a.w2_gs = _dev(w2_gs, "w2_gs", torch.float32).value
    a.inter_gs = None if inter_gs is None else _dev(inter_gs, "inter_gs", torch.float32).value
    a.out = None if out is None else _dev(out, "out", torch.bfloat16).value
    return a


def nvfp4_moe_forward(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales,
                      w2_gs, inter_gs, out, workspace, stream=None):
    """out [T, H] bf16 = the routed-expert MoE block (see include/nvfp4moe.h)."""
    a = _moe_args(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
                  inter_gs, out)
    _check(lib().nvfp4_moe_forward(ctypes.byref(a), _dev(workspace, "workspace", torch.uint8), workspace.numel(),
                                   _stream(stream)), "nvfp4_moe_forward")


def nvfp4_moe_forward_quantized(x_codes, x_scales, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs,
                                w2_codes, w2_scales, w2_gs, inter_gs, out, workspace, stream=None):
    """nvfp4_moe_forward on activations already in NVFP4: x_codes uint8
    [T, H/2] and row-major x_scales uint8 [T, H/16] made with the global scale
    x_gs (float32 [1], required)."""
    if x_gs is None:
        raise ValueError("x_gs (the global scale of the codes) is required")
    T, H = x_codes.shape[0], x_codes.shape[1] * 2
    if tuple(x_scales.shape) != (T, H // 16):
        raise ValueError(f"x_scales must be [{T}, {H // 16}] (row-major), got {tuple(x_scales.shape)}")
    a = _moe_args(None, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
                  inter_gs, out, x_shape=(T, H))
    _check(lib().nvfp4_moe_forward_quantized(ctypes.byref(a), _dev(x_codes, "x_codes", torch.uint8),
                                             _dev(x_scales, "x_scales", torch.uint8),
                                             _dev(workspace, "workspace", torch.uint8), workspace.numel(),
                                             _stream(stream)), "nvfp4_moe_forward_quantized")


def nvfp4_moe_forward_timed(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes,
                            w2_scales, w2_gs, inter_gs, out, workspace, events, stream=None):
    """nvfp4_moe_forward recording events[0..5] (torch.cuda.Event, timing
    enabled) before route, quantise+permute, L1, L2, combine and after combine."""
    a = _moe_args(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
                  inter_gs, out)
    if len(events) != 6:
        raise ValueError("events must hold 6 torch.cuda.Event objects")
    for e in events:
        if e.cuda_event == 0:           # torch creates the CUDA event on its first record()
            e.record()
    ev = (ctypes.c_void_p * 6)(*[e.cuda_event for e in events])
    _check(lib().nvfp4_moe_forward_timed(ctypes.byref(a), _dev(workspace, "workspace", torch.uint8),
                                         workspace.numel(), _stream(stream), ev), "nvfp4_moe_forward_timed")


def nvfp4_moe_forward_noalloc(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes,
                              w2_scales, w2_gs, inter_gs, out, stream=None):
    """nvfp4_moe_forward with the library's own fixed 32 MiB device scratch
    instead of a workspace (for callers that cannot allocate device memory);
    calls that overlap on the GPU race for that scratch."""
    a = _moe_args(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
                  inter_gs, out)
    _check(lib().nvfp4_moe_forward_noalloc(ctypes.byref(a), _stream(stream)), "nvfp4_moe_forward_noalloc")


def nvfp4_moe_calibrate(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales,
                        w2_gs, inter_gs_out, workspace, stream=None):
    """inter_gs_out [E] = warmup intermediate global scales from the batch (x, topk_ids)."""
    a = _moe_args(x, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs, w2_codes, w2_scales, w2_gs,
                  None, None)
    _check(lib().nvfp4_moe_calibrate(ctypes.byref(a), _dev(inter_gs_out, "inter_gs_out", torch.float32),
                                     _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)),
           "nvfp4_moe_calibrate")


def nvfp4_moe_route_debug(topk_ids, E, counts, padded_offsets, inv, workspace, stream=None):
    T, k = topk_ids.shape
    _check(lib().nvfp4_moe_route_debug(_dev(topk_ids, "topk_ids", torch.int32), T, k, E,
                                       _dev(counts, "counts", torch.int32),
                                       _dev(padded_offsets, "padded_offsets", torch.int32),
                                       _dev(inv, "inv", torch.int32), _dev(workspace, "workspace", torch.uint8),
                                       workspace.numel(), _stream(stream)), "nvfp4_moe_route_debug")


def nvfp4_moe_workspace_region(T, k, E, H, I, region):
    off, nbytes = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().nvfp4_moe_workspace_region(T, k, E, H, I, region, ctypes.byref(off), ctypes.byref(nbytes)),
           "nvfp4_moe_workspace_region")
    return off.value, nbytes.value


def nvfp4_moe_get_error(workspace, stream=None) -> int:
    """Reads and clears the workspace's device error word (synchronises the stream)."""
    err = ctypes.c_int32()
    _check(lib().nvfp4_moe_get_error(_dev(workspace, "workspace", torch.uint8), ctypes.byref(err), _stream(stream)),
           "nvfp4_moe_get_error")
    return err.value


NVFP4_SCORING_SOFTMAX = 0
NVFP4_SCORING_SIGMOID = 1


def nvfp4_moe_topk(logits, k, topk_ids, topk_weights, scoring=NVFP4_SCORING_SOFTMAX, stream=None):
    """Top-k router on the device: logits [T, E] fp32 -> topk_ids [T, k] int32,
    topk_weights [T, k] fp32 (renormalised softmax or sigmoid of the selection)."""
    T, E = logits.shape
    _check(lib().nvfp4_moe_topk(_dev(logits, "logits", torch.float32), T, E, k, scoring,
                                _dev(topk_ids, "topk_ids", torch.int32),
                                _dev(topk_weights, "topk_weights", torch.float32), _stream(stream)),
           "nvfp4_moe_topk")


def nvfp4_moe_topk_shared(logits, k, num_shared, topk_ids, topk_weights, scoring=NVFP4_SCORING_SOFTMAX,
                          stream=None):
    """The router with shared experts folded in: logits [T, E] fp32 ->
    topk_ids / topk_weights [T, k + num_shared], the k routed slots as
    nvfp4_moe_topk writes them, then slot k + i = expert E + i, weight 1."""
    T, E = logits.shape
    if tuple(topk_ids.shape) != (T, k + num_shared) or tuple(topk_weights.shape) != (T, k + num_shared):
        raise ValueError(f"topk_ids / topk_weights must be [{T}, {k + num_shared}]")
    _check(lib().nvfp4_moe_topk_shared(_dev(logits, "logits", torch.float32), T, E, k, scoring, num_shared,
                                       _dev(topk_ids, "topk_ids", torch.int32),
                                       _dev(topk_weights, "topk_weights", torch.float32), _stream(stream)),
           "nvfp4_moe_topk_shared")


def nvfp4_fp4_mma_ceiling(bn, iters, cycles, err=None, stream=None):
    """Tensor-core ceiling probe: cycles.numel() blocks each issue `iters`
    k-tiles of four FP4 MMAs (M=128, N=bn, K=64); cycles (int64, device)
    receives each block's issue-to-completion SM cycles."""
    _check(lib().nvfp4_fp4_mma_ceiling(bn, iters, cycles.numel(), _dev(cycles, "cycles", torch.int64),
                                       None if err is None else _dev(err, "err", torch.int32), _stream(stream)),
           "nvfp4_fp4_mma_ceiling")


def nvfp4_tma_stream_ceiling(matrix, work_tiles, stages=4, err=None, stream=None):
    """TMA streaming probe over a uint8 CUDA matrix [rows, row_bytes]: moves
    work_tiles * 256 * row_bytes bytes into shared memory (see
    nvfp4_tma_stream_ceiling in include/nvfp4moe.h)."""
    rows, row_bytes = matrix.shape
    _check(lib().nvfp4_tma_stream_ceiling(_dev(matrix, "matrix", torch.uint8), rows, row_bytes, work_tiles, stages,
                                          None if err is None else _dev(err, "err", torch.int32), _stream(stream)),
           "nvfp4_tma_stream_ceiling")


def nvfp4_moe_plan(T, k, E, H, I):
    """(fused_l1_l2: bool, pair_mode: 0 | 1 | 2) of the forward's execution
    plan (see nvfp4_moe_plan in include/nvfp4moe.h)."""
    f, pt = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().nvfp4_moe_plan(T, k, E, H, I, ctypes.byref(f), ctypes.byref(pt)), "nvfp4_moe_plan")
    return bool(f.value), int(pt.value)


def nvfp4_amax(x, amax_out, stream=None):
    """amax_out (device float [1]) = max|x| of a bf16 CUDA tensor."""
    _check(lib().nvfp4_amax(_dev(x, "x", torch.bfloat16), x.numel(), _dev(amax_out, "amax_out", torch.float32),
                            _stream(stream)), "nvfp4_amax")


def nvfp4_debug_bounded_wait(flag, target, err, stream=None):
    """Runs the fused launch's bounded device wait on flag (int32 [1], device)
    until flag >= target; err (int32 [1], device) receives NVFP4_ERR_TIMEOUT
    if the wait gives up (after 2 s)."""
    _check(lib().nvfp4_debug_bounded_wait(_dev(flag, "flag", torch.int32), target, _dev(err, "err", torch.int32),
                                          _stream(stream)), "nvfp4_debug_bounded_wait")
