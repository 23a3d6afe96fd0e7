"""ctypes marshalling for oracle.c (the CPU reference).

TEST INFRASTRUCTURE ONLY.  Every numeric step is in oracle.c; this file only
converts numpy arrays to pointers and back.  See oracle.c for the passages of
"nvfp4-megamoe-kernel / CURRENT_BUG.md" each step follows and for the
readings R1..R8 taken where the page is silent.

Parity status of each entry point (what pins it lives in tests/test_oracle_*.py):
  e2m1_encode / e2m1_decode      pinned (hand table, ml_dtypes, exhaustive)
  e4m3_encode / e4m3_decode      pinned (hand table, ml_dtypes, exhaustive)
  global_scale_from_amax         pinned (closed form at powers of two, amax*gs)
  quantize_bf16 / quantize_f32   pinned (worked block, invariants, ml_dtypes)
  dequantize                     pinned (exact values, error bound)
  route                          pinned (numpy stable argsort, bincount)
  gemm                           pinned (numpy matmul on dequantised operands)
  moe_forward                    pinned (per-token brute force, dense reduction)
  moe_warmup_inter_gs            pinned (brute-force amax of h)
  topk                           pinned (numpy stable sort, torch softmax / sigmoid;
                                 shared slots: the folded chain equals the routed
                                 chain plus the one-expert dense chain)
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


class MoeArgs(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
        ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("x", ctypes.c_void_p), ("topk_ids", ctypes.c_void_p), ("topk_weights", ctypes.c_void_p),
        ("x_gs", ctypes.c_float),
        ("w13_codes", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p), ("w13_gs", ctypes.c_void_p),
        ("w2_codes", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p), ("w2_gs", ctypes.c_void_p),
        ("inter_gs", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("h", ctypes.c_void_p), ("h_codes", ctypes.c_void_p),
        ("h_scales", ctypes.c_void_p), ("y", ctypes.c_void_p), ("h_amax", ctypes.c_void_p),
        ("x_codes", ctypes.c_void_p), ("x_scales", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_float
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_global_scale_from_amax.argtypes = [ctypes.c_float]
        L.oracle_global_scale_from_amax.restype = ctypes.c_float
        L.oracle_amax_bf16.argtypes = [P, i64]
        L.oracle_amax_bf16.restype = ctypes.c_float
        L.oracle_amax_f32.argtypes = [P, i64]
        L.oracle_amax_f32.restype = ctypes.c_float
        L.oracle_quantize_bf16.argtypes = [P, i64, i64, i64, ctypes.c_float, P, P]
        L.oracle_quantize_f32.argtypes = [P, i64, i64, i64, ctypes.c_float, P, P]
        L.oracle_dequantize.argtypes = [P, P, i64, i64, ctypes.c_float, P]
        L.oracle_route.argtypes = [P, i64, ctypes.c_int, P, P, P, P, P]
        L.oracle_route.restype = ctypes.c_int
        L.oracle_gemm.argtypes = [P, P, ctypes.c_float, i64, P, P, P, P, ctypes.c_int, i64, i64, P]
        L.oracle_moe_forward.argtypes = [ctypes.POINTER(MoeArgs)]
        L.oracle_moe_forward.restype = ctypes.c_int
        L.oracle_moe_warmup_inter_gs.argtypes = [ctypes.POINTER(MoeArgs), P]
        L.oracle_moe_warmup_inter_gs.restype = ctypes.c_int
        L.oracle_topk.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_topk_shared.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


def e2m1_encode(v: float) -> int:
    return int(lib().oracle_e2m1_encode(float(v)))


def e2m1_decode(c: int) -> float:
    return float(lib().oracle_e2m1_decode(int(c)))


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(b: int) -> float:
    return float(lib().oracle_e4m3_decode(int(b)))


def global_scale_from_amax(amax: float) -> np.float32:
    return np.float32(lib().oracle_global_scale_from_amax(float(amax)))


def amax_bf16(x_bits: np.ndarray) -> np.float32:
    x = _c(x_bits, np.uint16)
    return np.float32(lib().oracle_amax_bf16(_ptr(x), x.size))


def amax_f32(x: np.ndarray) -> np.float32:
    x = _c(x, np.float32)
    return np.float32(lib().oracle_amax_f32(_ptr(x), x.size))


def global_scale_bf16(x_bits: np.ndarray) -> np.float32:
    return global_scale_from_amax(amax_bf16(x_bits))


def quantize_bf16(x_bits: np.ndarray, gs: float):
    """x_bits: uint16 [rows, cols] bf16 bit patterns -> (codes u8 [rows, cols/2], scales u8 [rows, cols/16])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    assert cols % 16 == 0
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    lib().oracle_quantize_bf16(_ptr(x), rows, cols, cols, float(np.float32(gs)), _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_f32(x: np.ndarray, gs: float):
    x = _c(x, np.float32)
    rows, cols = x.shape
    assert cols % 16 == 0
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    lib().oracle_quantize_f32(_ptr(x), rows, cols, cols, float(np.float32(gs)), _ptr(codes), _ptr(scales))
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, gs: float) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    rows, half = codes.shape
    out = np.empty((rows, half * 2), np.float32)
    lib().oracle_dequantize(_ptr(codes), _ptr(scales), rows, half * 2, float(np.float32(gs)), _ptr(out))
    return out


def route(ids: np.ndarray, E: int):
    """Returns dict(counts, offsets, padded_offsets, rank, pos_padded, bad)."""
    ids = _c(ids, np.int32).reshape(-1)
    R = ids.size
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    poff = np.empty(E + 1, np.int32)
    rank = np.empty(R, np.int32)
    posp = np.empty(R, np.int32)
    bad = lib().oracle_route(_ptr(ids), R, E, _ptr(counts), _ptr(offsets), _ptr(poff), _ptr(rank), _ptr(posp))
    return dict(counts=counts, offsets=offsets, padded_offsets=poff, rank=rank, pos_padded=posp, bad=bad)


def gemm(a_codes, a_scales, a_gs, b_codes, b_scales, b_gs, seg_end=None) -> np.ndarray:
    a_codes = _c(a_codes, np.uint8)
    a_scales = _c(a_scales, np.uint8)
    b_codes = _c(b_codes, np.uint8)
    b_scales = _c(b_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    b_gs = np.atleast_1d(_c(b_gs, np.float32))
    if seg_end is None:
        seg_end = [N]
    seg = _c(seg_end, np.int64)
    assert seg.size == b_gs.size and seg[-1] == N
    out = np.empty((M, N), np.float32)
    lib().oracle_gemm(_ptr(a_codes), _ptr(a_scales), float(np.float32(a_gs)), M, _ptr(b_codes),
                      _ptr(b_scales), _ptr(b_gs), _ptr(seg), seg.size, N, K, _ptr(out))
    return out


def _moe_args(x_bits, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs,
              w2_codes, w2_scales, w2_gs, inter_gs, keep, x_codes=None, x_scales=None):
    if x_codes is not None:                 # activations given already quantised
        xc, xsc = _c(x_codes, np.uint8), _c(x_scales, np.uint8)
        T, H = xc.shape[0], xc.shape[1] * 2
        keep.append((xc, xsc))
        x = np.zeros((T, H), np.uint16)      # not read
    else:
        x = _c(x_bits, np.uint16)
        T, H = x.shape
    ids = _c(topk_ids, np.int32)
    k = ids.shape[1]
    wts = _c(topk_weights, np.float32)
    w13_codes = _c(w13_codes, np.uint8)
    E = w13_codes.shape[0]
    I = w13_codes.shape[1] // 2
    arrays = dict(x=x, ids=ids, wts=wts, w13_codes=w13_codes, w13_scales=_c(w13_scales, np.uint8),
                  w13_gs=_c(w13_gs, np.float32).reshape(E, 2), w2_codes=_c(w2_codes, np.uint8),
                  w2_scales=_c(w2_scales, np.uint8), w2_gs=_c(w2_gs, np.float32).reshape(E),
                  inter_gs=None if inter_gs is None else _c(inter_gs, np.float32).reshape(E))
    keep.append(arrays)
    a = MoeArgs()
    a.T, a.H, a.I, a.E, a.k = T, H, I, E, k
    a.x, a.topk_ids, a.topk_weights = _ptr(x), _ptr(ids), _ptr(wts)
    a.x_gs = float(np.float32(x_gs))
    a.w13_codes, a.w13_scales, a.w13_gs = _ptr(arrays["w13_codes"]), _ptr(arrays["w13_scales"]), _ptr(arrays["w13_gs"])
    a.w2_codes, a.w2_scales, a.w2_gs = _ptr(arrays["w2_codes"]), _ptr(arrays["w2_scales"]), _ptr(arrays["w2_gs"])
    a.inter_gs = _ptr(arrays["inter_gs"])
    if x_codes is not None:
        a.x_codes, a.x_scales = _ptr(xc), _ptr(xsc)
    return a, (T, H, I, E, k)


def moe_forward(x_bits, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs,
                w2_codes, w2_scales, w2_gs, inter_gs, intermediates=False, x_codes=None, x_scales=None):
    """Full chain.  Weights are given with canonical row-major scales:
    w13_codes [E, 2I, H/2], w13_scales [E, 2I, H/16], w2_codes [E, H, I/2],
    w2_scales [E, H, I/16].  With x_codes / x_scales ([T, H/2], [T, H/16])
    the activations are taken as already quantised with x_gs (x_bits is
    ignored).  Returns out fp32 [T, H] (and, with intermediates=True, a dict
    of h / h_codes / h_scales / y in slot order)."""
    keep = []
    a, (T, H, I, E, k) = _moe_args(x_bits, topk_ids, topk_weights, x_gs, w13_codes, w13_scales,
                                   w13_gs, w2_codes, w2_scales, w2_gs, inter_gs, keep, x_codes, x_scales)
    out = np.zeros((T, H), np.float32)
    a.out = _ptr(out)
    inter = None
    if intermediates:
        R = T * k
        inter = dict(h=np.zeros((R, I), np.float32), h_codes=np.zeros((R, I // 2), np.uint8),
                     h_scales=np.zeros((R, I // 16), np.uint8), y=np.zeros((R, H), np.float32),
                     h_amax=np.zeros(E, np.float32))
        a.h, a.h_codes, a.h_scales = _ptr(inter["h"]), _ptr(inter["h_codes"]), _ptr(inter["h_scales"])
        a.y, a.h_amax = _ptr(inter["y"]), _ptr(inter["h_amax"])
    bad = lib().oracle_moe_forward(ctypes.byref(a))
    if intermediates:
        inter["bad"] = bad
        return out, inter
    return out


def moe_warmup_inter_gs(x_bits, topk_ids, topk_weights, x_gs, w13_codes, w13_scales, w13_gs,
                        w2_codes, w2_scales, w2_gs) -> np.ndarray:
    keep = []
    a, (T, H, I, E, k) = _moe_args(x_bits, topk_ids, topk_weights, x_gs, w13_codes, w13_scales,
                                   w13_gs, w2_codes, w2_scales, w2_gs, None, keep)
    out = np.empty(E, np.float32)
    lib().oracle_moe_warmup_inter_gs(ctypes.byref(a), _ptr(out))
    return out


def topk(logits: np.ndarray, k: int, scoring: str = "softmax", num_shared: int = 0):
    """(ids int32 [T, k + num_shared], weights fp32 [T, k + num_shared]) from
    router logits [T, E] fp32; slot k + i is shared expert E + i, weight 1."""
    l = _c(logits, np.float32)
    T, E = l.shape
    assert 1 <= k <= min(E, 32) and 0 <= num_shared and k + num_shared <= 32
    ids = np.empty((T, k + num_shared), np.int32)
    w = np.empty((T, k + num_shared), np.float32)
    lib().oracle_topk_shared(_ptr(l), T, E, k, {"softmax": 0, "sigmoid": 1}[scoring], num_shared, _ptr(ids), _ptr(w))
    return ids, w
