"""CPU oracle for the fused MoE expert-FFN forward -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the CUDA library under ``mixture_experts_ffn_planner_b200``)
shares no code with it and never calls it.

The arithmetic lives in ``oracle.c`` (plain C, double accumulation); this file
only compiles it on demand and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no FP contraction)."""
    stale = (not os.path.exists(_LIB)
             or os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_double.restype = ctypes.c_double
        lib.orc_double_to_bf16.argtypes = [ctypes.c_double]
        lib.orc_double_to_bf16.restype = ctypes.c_uint16
        lib.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_to_double.restype = ctypes.c_double
        lib.orc_double_to_e4m3.argtypes = [ctypes.c_double]
        lib.orc_double_to_e4m3.restype = ctypes.c_uint8
        lib.orc_e8m0_to_double.argtypes = [ctypes.c_uint8]
        lib.orc_e8m0_to_double.restype = ctypes.c_double
        lib.orc_mx_scale_byte.argtypes = [ctypes.c_float]
        lib.orc_mx_scale_byte.restype = ctypes.c_uint8
        lib.orc_mx_quantize.argtypes = [P, I64, P, P]
        lib.orc_mx_quantize.restype = None
        lib.orc_align_capacity.argtypes = [I, I, I, I]
        lib.orc_align_capacity.restype = I64
        lib.orc_moe_align.argtypes = [P, I, I, I, I, P, P, P, I64]
        lib.orc_moe_align.restype = I
        lib.orc_route_topk.argtypes = [P, P, I, I, I, I, P, P]
        lib.orc_route_topk.restype = I
        lib.orc_pack_scales_bytes.argtypes = [I, I, I]
        lib.orc_pack_scales_bytes.restype = I64
        lib.orc_pack_scales_blocked.argtypes = [P, P, I, I, I]
        lib.orc_pack_scales_blocked.restype = None
        lib.orc_unpack_scales_blocked.argtypes = [P, P, I, I, I]
        lib.orc_unpack_scales_blocked.restype = None
        lib.orc_fused_moe_bf16.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, P, I]
        lib.orc_fused_moe_bf16.restype = None
        lib.orc_fused_moe_mxfp8.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, I, P, P, I]
        lib.orc_fused_moe_mxfp8.restype = None
        lib.orc_fused_moe_mxfp4.argtypes = lib.orc_fused_moe_mxfp8.argtypes
        lib.orc_fused_moe_mxfp4.restype = None
        lib.orc_mx_intermediate.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, I, I]
        lib.orc_mx_intermediate.restype = None
        lib.orc_e2m1_to_double.argtypes = [ctypes.c_uint8]
        lib.orc_e2m1_to_double.restype = ctypes.c_double
        lib.orc_max_threads.argtypes = []
        lib.orc_max_threads.restype = I
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ---- scalar formats -------------------------------------------------------
def bf16_to_double(bits: int) -> float:
    return _load().orc_bf16_to_double(int(bits))


def double_to_bf16(x: float) -> int:
    return int(_load().orc_double_to_bf16(float(x)))


def e4m3_to_double(code: int) -> float:
    return _load().orc_e4m3_to_double(int(code))


def double_to_e4m3(x: float) -> int:
    return int(_load().orc_double_to_e4m3(float(x)))


def e8m0_to_double(code: int) -> float:
    return _load().orc_e8m0_to_double(int(code))


def mx_scale_byte(amax: float) -> int:
    return int(_load().orc_mx_scale_byte(float(amax)))


def mx_quantize(v: np.ndarray):
    """fp32 values (last dim a multiple of 32) -> (e4m3 codes, e8m0 scales)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    assert v.shape[-1] % 32 == 0
    codes = np.empty(v.shape, dtype=np.uint8)
    scales = np.empty(v.shape[:-1] + (v.shape[-1] // 32,), dtype=np.uint8)
    _load().orc_mx_quantize(_ptr(v), v.size, _ptr(codes), _ptr(scales))
    return codes, scales


# ---- planner --------------------------------------------------------------
def align_capacity(T: int, top_k: int, E: int, block_m: int) -> int:
    return int(_load().orc_align_capacity(T, top_k, E, block_m))


def moe_align(topk_ids: np.ndarray, E: int, block_m: int, capacity: int | None = None):
    """Returns (sorted_token_ids, expert_ids, num_tokens_post_padded)."""
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, k = ids.shape
    cap = align_capacity(T, k, E, block_m) if capacity is None else int(capacity)
    sorted_ids = np.empty(cap, dtype=np.int32)
    expert_ids = np.empty((cap + block_m - 1) // block_m, dtype=np.int32)
    ntpp = np.zeros(1, dtype=np.int32)
    rc = _load().orc_moe_align(_ptr(ids), T, k, E, block_m, _ptr(sorted_ids), _ptr(expert_ids),
                               _ptr(ntpp), cap)
    if rc != 0:
        raise RuntimeError(f"oracle moe_align failed ({rc})")
    return sorted_ids, expert_ids, int(ntpp[0])


def route_topk(logits: np.ndarray, top_k: int, bias: np.ndarray | None = None, n_shared: int = 0):
    """Router: (T, E) fp32 logits (+ optional (E,) fp32 bias) -> (topk_ids (T, top_k + n_shared) int32,
    topk_weights (T, top_k + n_shared) float64).  Ranking on the fp32 score logits + bias, ties to
    the lower expert; weights are the renormalised softmax over the kept experts; then n_shared
    routes to the shared experts E, E+1, ... with weight 1."""
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    if b is not None and b.shape != (E,):
        raise ValueError("bias must have shape (E,)")
    kk = top_k + n_shared
    ids = np.empty((T, kk), dtype=np.int32)
    w = np.empty((T, kk), dtype=np.float64)
    rc = _load().orc_route_topk(_ptr(lg), None if b is None else _ptr(b), T, E, top_k, n_shared, _ptr(ids),
                                _ptr(w))
    if rc != 0:
        raise RuntimeError(f"oracle route_topk failed ({rc})")
    return ids, w


# ---- blocked scales -------------------------------------------------------
def pack_scales_blocked(s: np.ndarray) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.uint8)
    E, MN, KS = s.shape
    out = np.empty(int(_load().orc_pack_scales_bytes(E, MN, KS)), dtype=np.uint8)
    _load().orc_pack_scales_blocked(_ptr(s), _ptr(out), E, MN, KS)
    return out


def unpack_scales_blocked(b: np.ndarray, E: int, MN: int, KS: int) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty((E, MN, KS), dtype=np.uint8)
    _load().orc_unpack_scales_blocked(_ptr(b), _ptr(out), E, MN, KS)
    return out


# ---- expert FFN -----------------------------------------------------------
def _tokens_arg(tokens, T):
    if tokens is None:
        return None, T
    t = np.ascontiguousarray(tokens, dtype=np.int32)
    assert t.ndim == 1 and (t.size == 0 or (t.min() >= 0 and t.max() < T))
    return t, int(t.size)


def fused_moe_bf16(x, w1, w2, topk_ids, topk_weights, tokens=None, nthreads: int = 0, unrounded: bool = False):
    """x (T,K) uint16 bf16 bits, w1 (E,N,K), w2 (E,K,N/2) -> out (T,K) uint16 bits.

    Rows of tokens not listed in ``tokens`` are left zero.  With
    ``unrounded=True`` also returns out before its final bf16 rounding
    (float64, (T, K))."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w1 = np.ascontiguousarray(w1, dtype=np.uint16)
    w2 = np.ascontiguousarray(w2, dtype=np.uint16)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    tw = np.ascontiguousarray(topk_weights, dtype=np.float32)
    T, K = x.shape
    E, N, K1 = w1.shape
    assert K1 == K and w2.shape == (E, K, N // 2)
    top_k = ids.shape[1]
    t, n = _tokens_arg(tokens, T)
    out = np.zeros((T, K), dtype=np.uint16)
    f64 = np.zeros((T, K), dtype=np.float64) if unrounded else None
    _load().orc_fused_moe_bf16(_ptr(x), _ptr(w1), _ptr(w2), _ptr(ids), _ptr(tw), T, K, N, E, top_k,
                               None if t is None else _ptr(t), n, _ptr(out),
                               None if f64 is None else _ptr(f64), int(nthreads))
    return (out, f64) if unrounded else out


def fused_moe_mxfp8(x, x_scales, w1, w1_scales, w2, w2_scales, topk_ids, topk_weights,
                    tokens=None, nthreads: int = 0, unrounded: bool = False):
    """All scales ROW-MAJOR: x_scales (T,K/32), w1_scales (E,N,K/32), w2_scales (E,K,N/64).

    With ``unrounded=True`` also returns out before its final bf16 rounding."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (x, x_scales, w1, w1_scales, w2, w2_scales)]
    x, xs, w1, s1, w2, s2 = arrs
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    tw = np.ascontiguousarray(topk_weights, dtype=np.float32)
    T, K = x.shape
    E, N, _ = w1.shape
    assert xs.shape == (T, K // 32) and s1.shape == (E, N, K // 32)
    assert w2.shape == (E, K, N // 2) and s2.shape == (E, K, N // 64)
    top_k = ids.shape[1]
    t, n = _tokens_arg(tokens, T)
    out = np.zeros((T, K), dtype=np.uint16)
    f64 = np.zeros((T, K), dtype=np.float64) if unrounded else None
    _load().orc_fused_moe_mxfp8(_ptr(x), _ptr(xs), _ptr(w1), _ptr(s1), _ptr(w2), _ptr(s2), _ptr(ids),
                                _ptr(tw), T, K, N, E, top_k, None if t is None else _ptr(t), n,
                                _ptr(out), None if f64 is None else _ptr(f64), int(nthreads))
    return (out, f64) if unrounded else out


def fused_moe_mxfp4(x, x_scales, w1, w1_scales, w2, w2_scales, topk_ids, topk_weights,
                    tokens=None, nthreads: int = 0, unrounded: bool = False):
    """mxfp8 activations, MXFP4 weights: w1 (E, N, K/2) and w2 (E, K, N/4) packed e2m1 codes
    (even index in the low nibble); scales ROW-MAJOR as for fused_moe_mxfp8."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (x, x_scales, w1, w1_scales, w2, w2_scales)]
    x, xs, w1, s1, w2, s2 = arrs
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    tw = np.ascontiguousarray(topk_weights, dtype=np.float32)
    T, K = x.shape
    E, N, Kh = w1.shape
    assert Kh * 2 == K and xs.shape == (T, K // 32) and s1.shape == (E, N, K // 32)
    assert w2.shape == (E, K, N // 4) and s2.shape == (E, K, N // 64)
    top_k = ids.shape[1]
    t, n = _tokens_arg(tokens, T)
    out = np.zeros((T, K), dtype=np.uint16)
    f64 = np.zeros((T, K), dtype=np.float64) if unrounded else None
    _load().orc_fused_moe_mxfp4(_ptr(x), _ptr(xs), _ptr(w1), _ptr(s1), _ptr(w2), _ptr(s2), _ptr(ids),
                                _ptr(tw), T, K, N, E, top_k, None if t is None else _ptr(t), n,
                                _ptr(out), None if f64 is None else _ptr(f64), int(nthreads))
    return (out, f64) if unrounded else out


def mx_intermediate(x, x_scales, w1, w1_scales, topk_ids, tokens=None, nthreads: int = 0, fp4: bool = False,
                    out=None):
    """The fp32 SwiGLU intermediate of the mxfp8 forward (MXFP4 weights with ``fp4``) before its
    requant: float32 (n, top_k, N/2) for the n listed tokens (all T when ``tokens`` is None), routes in
    top-k order; a route to an expert outside [0, E) gives a zero row.  Scales row-major as for
    fused_moe_mxfp8; w1 (E, N, K) e4m3 codes, or (E, N, K/2) packed e2m1 codes with ``fp4``."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (x, x_scales, w1, w1_scales)]
    x, xs, w1, s1 = arrs
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, K = x.shape
    E, N, Kw = w1.shape
    assert Kw * (2 if fp4 else 1) == K and xs.shape == (T, K // 32) and s1.shape == (E, N, K // 32)
    top_k = ids.shape[1]
    t, n = _tokens_arg(tokens, T)
    act = np.empty((n, top_k, N // 2), dtype=np.float32) if out is None else out
    assert act.shape == (n, top_k, N // 2) and act.dtype == np.float32 and act.flags["C_CONTIGUOUS"]
    _load().orc_mx_intermediate(_ptr(x), _ptr(xs), _ptr(w1), _ptr(s1), _ptr(ids), T, K, N, E, top_k,
                                None if t is None else _ptr(t), n, _ptr(act), int(nthreads), int(bool(fp4)))
    return act


def e2m1_to_double(code: int) -> float:
    return float(_load().orc_e2m1_to_double(code))


def max_threads() -> int:
    return int(_load().orc_max_threads())
