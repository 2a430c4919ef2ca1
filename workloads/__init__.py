"""Seeded synthetic inputs for the fused MoE expert-FFN forward.

This module is shared by the test suite and ``bench.py``.  It draws random
numbers and prepares them the way a caller would hand them to the op; it holds
none of the op's own arithmetic (no planner, no GEMM, no SwiGLU, no requant of
the intermediate, no scale packing).

Workloads (the five shapes the benchmark and tests are quoted on):

=====  =======  ====  ====  ====  =====  =======  ===========================
name   dtype    K     N     E     top_k  block_m  T
=====  =======  ====  ====  ====  =====  =======  ===========================
C1     bf16     1024  1024  8     2      64       64
C2     bf16     4096  4096  256   6      128      64, 256
C3     mxfp8    4096  4096  288   8      128      64 ... 8192
C4     mxfp8    7168  6144  384   6      128      1024 ... 8192
C5     bf16     4096  512   128   8      128      1, 8, 64, 512, 8192 (Zipf bias)
C3F4   mxfp4    4096  4096  288   8      128      64 ... 8192 (C3 with MXFP4 weights)
C4F4   mxfp4    7168  6144  384   6      128      1024 ... 8192 (C4 with MXFP4 weights)
=====  =======  ====  ====  ====  =====  =======  ===========================

The two F4 workloads draw the same fp32 tensors as C3 / C4 and quantise the
weights to MXFP4 (e2m1 values, e8m0 scale per 32 along K, two values per byte,
the even-indexed value in the low nibble) instead of mxfp8; activations stay
mxfp8.

Recipe (all fp32 draws from numpy PCG64 streams keyed by
``SeedSequence([seed, workload, tensor, expert])``):

* ``x ~ N(0, 1)``; ``w1[e] ~ N(0, 1/sqrt(K))``; ``w2[e] ~ N(0, 1/sqrt(N/2))``.
* bf16 inputs: fp32 -> bf16 round-to-nearest-even.
* mxfp8 inputs: the caller-side OCP MX quantiser (block 32 along the
  contraction dimension, e4m3 values, e8m0 scales) -- the pages leave input
  quantisation to the caller ("Prime Flash MoE: Fused MoE Kernels for
  Blackwell", Scale layout (mxfp8)); weight scales are returned row-major and
  the caller packs them.
* routing: logits ``~ N(0, 1)`` (T, E) fp32, plus on C5 a per-expert bias
  ``-s * ln(rank_e)`` with ``rank`` a seeded permutation of 1..E and s = 1.2;
  softmax in float64, top-k by descending probability (ties to the lower
  expert index), weights renormalised to sum to one, stored fp32.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import os

import numpy as np

DEFAULT_SEED = 20261202

_WORKLOADS = {
    "C1": dict(dtype="bf16", K=1024, N=1024, E=8, top_k=2, block_m=64, Ts=(64,), zipf_s=None),
    "C2": dict(dtype="bf16", K=4096, N=4096, E=256, top_k=6, block_m=128, Ts=(64, 256), zipf_s=None),
    "C3": dict(dtype="mxfp8", K=4096, N=4096, E=288, top_k=8, block_m=128,
               Ts=(64, 256, 1024, 2048, 4096, 8192), zipf_s=None),
    "C4": dict(dtype="mxfp8", K=7168, N=6144, E=384, top_k=6, block_m=128,
               Ts=(1024, 2048, 4096, 8192), zipf_s=None),
    "C5": dict(dtype="bf16", K=4096, N=512, E=128, top_k=8, block_m=128,
               Ts=(1, 8, 64, 512, 8192), zipf_s=1.2),
    "C3F4": dict(dtype="mxfp4", K=4096, N=4096, E=288, top_k=8, block_m=128,
                 Ts=(64, 256, 1024, 2048, 4096, 8192), zipf_s=None),
    "C4F4": dict(dtype="mxfp4", K=7168, N=6144, E=384, top_k=6, block_m=128,
                 Ts=(1024, 2048, 4096, 8192), zipf_s=None),
}
# random streams: the F4 workloads share their base workload's draws
_STREAM_KEY = {"C1": 1, "C2": 2, "C3": 3, "C4": 4, "C5": 5, "C3F4": 3, "C4F4": 4}
_TENSOR_IDS = {"x": 1, "w1": 2, "w2": 3, "logits": 4, "rank": 5}


@dataclasses.dataclass(frozen=True)
class Shape:
    name: str
    dtype: str          # "bf16" | "mxfp8"
    T: int
    K: int
    N: int              # fused gate+up width; intermediate I = N // 2
    E: int
    top_k: int
    block_m: int
    zipf_s: float | None = None

    @property
    def I(self) -> int:  # noqa: E743  (intermediate size, the pages' N // 2)
        return self.N // 2

    @property
    def R(self) -> int:
        return self.T * self.top_k


def workload_names():
    return list(_WORKLOADS)


def token_counts(name: str):
    return tuple(_WORKLOADS[name]["Ts"])


def shape(name: str, T: int | None = None, **override) -> Shape:
    """The named workload at token count T (default: its largest)."""
    w = dict(_WORKLOADS[name])
    Ts = w.pop("Ts")
    w.update(override)
    return Shape(name=name, T=int(T if T is not None else Ts[-1]), **w)


def _rng(seed: int, sh: Shape, tensor: str, expert: int = 0) -> np.random.Generator:
    key = [int(seed), _STREAM_KEY.get(sh.name, 0), _TENSOR_IDS[tensor],
           int(expert), int(sh.T) if tensor in ("x", "logits") else 0]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def _threads(n: int | None) -> int:
    return int(n) if n else max(1, min(32, os.cpu_count() or 1))


# ---------------------------------------------------------------------------
# caller-side conversions
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def mx_quantize_inputs(v: np.ndarray):
    """Caller-side OCP MX quantiser: (..., L) fp32 -> e4m3 codes (..., L), e8m0 (..., L/32).

    Scale 2^(floor(log2 amax) - 8) per block of 32 (8 = emax of e4m3; an all-zero block gets byte
    0), values multiplied by the inverse power of two in fp32, clamped to +-448 and rounded to e4m3
    by torch's float8_e4m3fn conversion (round to nearest even).  The elementwise passes run as
    torch CPU ops (multi-threaded); the per-block scale arithmetic in numpy."""
    import torch

    v = np.ascontiguousarray(v, dtype=np.float32)
    L = v.shape[-1]
    assert L % 32 == 0
    blk = torch.from_numpy(v).view(-1, 32)
    amax = blk.abs().amax(dim=1).numpy()
    _, ex = np.frexp(amax)                      # amax = m * 2^ex, 0.5 <= m < 1
    shared = ex.astype(np.int32) - 1 - 8        # floor(log2 amax) - emax(e4m3)
    shared = np.where(amax > 0, shared, -127)
    shared = np.clip(shared, -127, 127)
    mult = torch.from_numpy(np.ldexp(np.float32(1.0), (-shared).astype(np.int32)).astype(np.float32))
    scaled = (blk * mult[:, None]).clamp_(-448.0, 448.0)
    codes = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes.reshape(v.shape), (shared + 127).astype(np.uint8).reshape(v.shape[:-1] + (L // 32,))


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------
def routing(sh: Shape, seed: int = DEFAULT_SEED):
    """(topk_ids int32 (T, k), topk_weights fp32 (T, k))."""
    logits = _rng(seed, sh, "logits").standard_normal((sh.T, sh.E), dtype=np.float32).astype(np.float64)
    if sh.zipf_s:
        rank = _rng(seed, sh, "rank").permutation(sh.E) + 1
        logits = logits + (-float(sh.zipf_s) * np.log(rank.astype(np.float64)))[None, :]
    logits = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, : sh.top_k]
    w = np.take_along_axis(p, order, axis=1)
    w = w / w.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def router_logits(sh: Shape, seed: int = DEFAULT_SEED):
    """Router inputs: (logits fp32 (T, E), per-expert bias fp32 (E,) or None).  The same draws
    as `routing` (N(0,1) logits; on Zipf-skewed workloads bias_e = -s * ln(rank_e) over a
    seeded rank permutation), before any routing arithmetic."""
    logits = _rng(seed, sh, "logits").standard_normal((sh.T, sh.E), dtype=np.float32)
    bias = None
    if sh.zipf_s:
        rank = _rng(seed, sh, "rank").permutation(sh.E) + 1
        bias = (-float(sh.zipf_s) * np.log(rank.astype(np.float64))).astype(np.float32)
    return logits, bias


def x_f32(sh: Shape, seed: int = DEFAULT_SEED) -> np.ndarray:
    return _rng(seed, sh, "x").standard_normal((sh.T, sh.K), dtype=np.float32)


def expert_f32(sh: Shape, which: str, e: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """One expert's weights in fp32: w1[e] (N, K) or w2[e] (K, N/2)."""
    if which == "w1":
        rows, fan_in = sh.N, sh.K
    else:
        rows, fan_in = sh.K, sh.I
    v = _rng(seed, sh, which, e).standard_normal((rows, fan_in), dtype=np.float32)
    v *= np.float32(1.0 / np.sqrt(fan_in))
    return v


def _fill_experts(sh: Shape, which: str, fn, out_arrays, seed, threads):
    def job(e):
        fn(e, expert_f32(sh, which, e, seed), out_arrays)
    with cf.ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(job, range(sh.E)))


def bf16_weights(sh: Shape, which: str, seed: int = DEFAULT_SEED, threads: int | None = None) -> np.ndarray:
    rows, cols = (sh.N, sh.K) if which == "w1" else (sh.K, sh.I)
    out = np.empty((sh.E, rows, cols), dtype=np.uint16)

    def put(e, v, o):
        o[e] = f32_to_bf16_bits(v)
    _fill_experts(sh, which, put, out, seed, threads)
    return out


def mxfp8_weights(sh: Shape, which: str, seed: int = DEFAULT_SEED, threads: int | None = None):
    """(codes (E, rows, cols) u8, row-major scales (E, rows, cols/32) u8)."""
    rows, cols = (sh.N, sh.K) if which == "w1" else (sh.K, sh.I)
    codes = np.empty((sh.E, rows, cols), dtype=np.uint8)
    scales = np.empty((sh.E, rows, cols // 32), dtype=np.uint8)

    def put(e, v, o):
        c, s = mx_quantize_inputs(v)
        o[0][e] = c
        o[1][e] = s
    _fill_experts(sh, which, put, (codes, scales), seed, threads)
    return codes, scales


def bf16_inputs(sh: Shape, seed: int = DEFAULT_SEED, threads: int | None = None) -> dict:
    ids, tw = routing(sh, seed)
    return dict(x=f32_to_bf16_bits(x_f32(sh, seed)), w1=bf16_weights(sh, "w1", seed, threads),
                w2=bf16_weights(sh, "w2", seed, threads), topk_ids=ids, topk_weights=tw)


def mx_quantize_fp4(v: np.ndarray):
    """Caller-side OCP MX FP4 quantiser: (..., L) fp32 -> packed e2m1 codes (..., L/2) u8 (value
    2j in the low nibble of byte j) and e8m0 scales (..., L/32).  Shared scale
    2^(floor(log2 amax) - 2) (emax of e2m1 is 2); values rounded to the nearest e2m1 magnitude
    (0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even code, beyond 6 saturated; an all-zero block gets
    scale byte 0.  The code of a scaled magnitude m is the number of rounding boundaries it has
    passed: 0.25, 1.25, 2.5 and 5 round down on a tie (the lower code is even), 0.75, 1.75 and 3.5
    round up; the sign bit is 8.  Elementwise passes as torch CPU ops in float64 (exact)."""
    import torch

    v = np.ascontiguousarray(v, dtype=np.float32)
    L = v.shape[-1]
    assert L % 32 == 0
    blk = torch.from_numpy(v).view(-1, 32).double()
    amax = blk.abs().amax(dim=1).numpy()
    _, ex = np.frexp(amax)
    shared = np.where(amax > 0, ex.astype(np.int32) - 1 - 2, -127)
    shared = np.clip(shared, -127, 127)
    scaled = blk * torch.from_numpy(np.ldexp(1.0, -shared))[:, None]
    mag = scaled.abs()
    code = ((mag > 0.25).to(torch.uint8) + (mag >= 0.75) + (mag > 1.25) + (mag >= 1.75) + (mag > 2.5)
            + (mag >= 3.5) + (mag > 5.0))
    codes = (code | (torch.signbit(scaled).to(torch.uint8) << 3)).numpy().reshape(v.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    scales = (shared + 127).astype(np.uint8).reshape(v.shape[:-1] + (L // 32,))
    return packed, scales


def mxfp4_weights(sh: Shape, which: str, seed: int = DEFAULT_SEED, threads: int | None = None):
    """(packed e2m1 (E, rows, cols/2) u8, row-major scales (E, rows, cols/32) u8)."""
    rows, cols = (sh.N, sh.K) if which == "w1" else (sh.K, sh.I)
    codes = np.empty((sh.E, rows, cols // 2), dtype=np.uint8)
    scales = np.empty((sh.E, rows, cols // 32), dtype=np.uint8)

    def put(e, v, o):
        c, s = mx_quantize_fp4(v)
        o[0][e] = c
        o[1][e] = s
    _fill_experts(sh, which, put, (codes, scales), seed, threads)
    return codes, scales


def mxfp8_inputs(sh: Shape, seed: int = DEFAULT_SEED, threads: int | None = None) -> dict:
    ids, tw = routing(sh, seed)
    xq, xs = mx_quantize_inputs(x_f32(sh, seed))
    wq = mxfp4_weights if sh.dtype == "mxfp4" else mxfp8_weights
    w1, s1 = wq(sh, "w1", seed, threads)
    w2, s2 = wq(sh, "w2", seed, threads)
    return dict(x=xq, x_scales=xs, w1=w1, w1_scales=s1, w2=w2, w2_scales=s2, topk_ids=ids, topk_weights=tw)


def inputs(sh: Shape, seed: int = DEFAULT_SEED, threads: int | None = None) -> dict:
    return bf16_inputs(sh, seed, threads) if sh.dtype == "bf16" else mxfp8_inputs(sh, seed, threads)


def sample_tokens(sh: Shape, topk_ids: np.ndarray, n: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """A seeded token sample that always includes tokens routed to the most-
    and least-loaded (non-empty) experts."""
    n = min(int(n), sh.T)
    counts = np.bincount(topk_ids.reshape(-1), minlength=sh.E)
    used = np.nonzero(counts)[0]
    must = set()
    for e in (used[np.argmax(counts[used])], used[np.argmin(counts[used])]):
        rows = np.nonzero((topk_ids == e).any(axis=1))[0]
        must.add(int(rows[0]))
        must.add(int(rows[-1]))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 99, sh.T])))
    rest = [t for t in rng.permutation(sh.T).tolist() if t not in must]
    picked = sorted(list(must)[:n] + rest[: max(0, n - len(must))])
    return np.array(picked, dtype=np.int32)
