"""Python binding of the B200 fused MoE expert-FFN forward (``libmoe_ffn.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/moe_ffn.h``.  PyTorch supplies
device memory and streams.  There is no CPU or PyTorch fallback: if the
library cannot be built or loaded, every call raises.

Entry points (same names as the C ABI):

* ``moe_align`` -- routing planner: expert histogram, prefix sums over counts
  padded to ``block_m``, and the row-to-token map ("[RFC] Fused W8A8 MoE
  megakernel on H20", Design; "Prime Flash MoE: Fused MoE Kernels for
  Blackwell", API / Shapes).
* ``moe_route_align`` -- the router ahead of the planner: softmax over the
  experts, top-k, renormalised weights, then the planner on the kept ids
  ("Prime Flash MoE", Usage; "[RFC] Fused W8A8 MoE megakernel on H20",
  Results so far).
* ``fused_moe_bf16`` / ``fused_moe_mxfp8`` -- gather, gate/up GEMM, SwiGLU
  (mxfp8: on-chip requant of the intermediate), down GEMM and the top-k
  weighted reduction into ``out`` ("Prime Flash MoE", intro / API / Shapes).
* ``fused_moe_mxfp4`` -- the mxfp8 forward with MXFP4 (e2m1) weights, two
  values per byte (DeepGEMM #411 "SM90 FP8 x MXFP4 MegaMoE" operand pairing).
* ``pack_scales_blocked`` -- weight scales into 512-byte tiles of
  128 MN x 128 K ("Prime Flash MoE", Scale layout (mxfp8)).
* ``moe_ep_dispatch_plan`` / ``moe_ep_dispatch_pack`` / ``moe_ep_combine`` --
  the device work around an expert-parallel exchange (DeepGEMM #411 "SM90 FP8
  x MXFP4 MegaMoE", Summary: dispatch, routed experts, combine).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

from . import _build

__all__ = [
    "MoeError", "load", "moe_align", "moe_align_capacity", "moe_route_align", "fused_moe_bf16", "fused_moe_mxfp8",
    "fused_moe_mxfp4", "DTYPE_MXFP4",
    "pack_scales_blocked", "pack_scales_blocked_bytes", "moe_workspace_bytes", "moe_device_status",
    "Tuning", "DTYPE_BF16", "DTYPE_MXFP8", "LIB_PATH", "fused_moe_bf16_noalloc",
    "fused_moe_bf16_noalloc_max_workspace", "moe_ep_dispatch_plan", "moe_ep_dispatch_pack", "moe_ep_combine",
]

DTYPE_BF16 = 0
DTYPE_MXFP8 = 1
DTYPE_MXFP4 = 2
LIB_PATH = _build.LIB

_ERRORS = {-1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_ALIGNMENT",
           -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA", -6: "MOE_ERR_TIMEOUT"}


class MoeError(RuntimeError):
    """A C-ABI call returned a negative status."""

    def __init__(self, code: int, message: str):
        self.code = int(code)
        self.name = _ERRORS.get(self.code, f"status {code}")
        super().__init__(f"{self.name}: {message}")


class Tuning(ctypes.Structure):
    """``moe_tuning``: 0 in a field keeps the library's default."""
    _fields_ = [("stages", ctypes.c_int), ("num_ctas", ctypes.c_int),
                ("phase_events", ctypes.POINTER(ctypes.c_void_p)), ("wait_timeout_ns", ctypes.c_longlong),
                ("small_batch", ctypes.c_int)]

    @staticmethod
    def with_events(events, stages: int = 0, num_ctas: int = 0) -> "Tuning":
        """Tuning whose timing hook records the four given torch.cuda.Event objects."""
        for e in events:
            e.record()  # forces creation of the underlying cudaEvent_t
        arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
        t = Tuning(stages, num_ctas, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
        t._keep = arr
        return t


_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64

_SIGS = {
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_device_status": ([_P], _I),
    "moe_align_capacity": ([_I, _I, _I, _I], _I64),
    "moe_align": ([_P, _I, _I, _I, _I, _P, _P, _P, _I64, _P], _I),
    "moe_route_align": ([_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I64, _P], _I),
    "pack_scales_blocked_bytes": ([_I, _I, _I], _I64),
    "pack_scales_blocked": ([_P, _P, _I, _I, _I, _P], _I),
    "moe_workspace_bytes": ([_I, _I, _I, _I, _I, _I, _I], _I64),
    "fused_moe_bf16": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _P, _I64, _P, _P], _I),
    "fused_moe_mxfp8": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _P, _I64,
                         _P, _P], _I),
    "fused_moe_mxfp4": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _P, _I64,
                         _P, _P], _I),
    "fused_moe_bf16_noalloc_max_workspace": ([], _I64),
    "moe_ep_dispatch_plan": ([_P, _I, _I, _I, _I, _P, _P, _P], _I),
    "moe_ep_dispatch_pack": ([_P, _I64, _P, _I64, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P], _I),
    "moe_ep_combine": ([_P, _P, _I, _I, _I, _I, _P, _P, _P], _I),
    "fused_moe_bf16_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _P, _P], _I),
}


def load(build_if_stale: bool = True) -> ctypes.CDLL:
    """Loads libmoe_ffn.so (compiling it first if a source is newer)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if build_if_stale and _build.stale():
            try:
                _build.build()
            except Exception as exc:  # no toolchain: use the library that is there, if any
                if not os.path.exists(_build.LIB):
                    raise ImportError(f"libmoe_ffn.so is missing and could not be built: {exc}") from exc
        if not os.path.exists(_build.LIB):
            raise ImportError(f"libmoe_ffn.so not found at {_build.LIB}; run __graft_entry__.build()")
        lib = ctypes.CDLL(_build.LIB)
        for name, (args, res) in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def _check(rc: int):
    if rc != 0:
        msg = load().moe_last_error()
        raise MoeError(rc, msg.decode() if msg else "")


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


@contextlib.contextmanager
def _on_device(dev, stream):
    """Makes ``dev`` (the device of the call's tensors) the current CUDA device
    for the C call and yields the stream handle to launch on.

    The library launches on the current device and builds its TMA descriptors
    from the tensors' addresses, so a call whose tensors live on another
    device than the current one would read that device's memory from the
    wrong GPU.  ``stream``: None (the current stream of ``dev``), a
    ``torch.cuda.Stream`` (must belong to ``dev``) or a raw ``cudaStream_t``
    handle as an int (the caller vouches for its device)."""
    import torch

    if getattr(dev, "type", None) != "cuda":
        raise ValueError(f"tensors must be on a CUDA device, got {dev}")
    with torch.cuda.device(dev):
        if stream is None:
            handle = torch.cuda.current_stream(dev).cuda_stream
        elif hasattr(stream, "cuda_stream"):
            sdev = getattr(stream, "device", dev)
            if torch.device(sdev) != torch.device(dev):
                raise ValueError(f"stream belongs to {sdev} but the tensors are on {dev}")
            handle = stream.cuda_stream
        else:
            handle = int(stream)
        yield handle


def _need(t, name, dtypes, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _ffn_shapes(fmt: str, x, w1, w2, topk_weights, out, sorted_token_ids, expert_ids, num_tokens_post_padded,
                block_m: int, x_scales=None, w1_scales=None, w2_scales=None):
    """The C ABI takes its sizes from x and w1 and trusts every other buffer, so the shapes (and the
    device) of all of them are checked here before a launch: a short buffer would be read or written
    out of bounds by the kernels.  fmt: "bf16", "mxfp8" or "mxfp4" (packed weights, two per byte)."""
    if x.dim() != 2 or w1.dim() != 3:
        raise ValueError("x must be (T, K) and w1 (E, N, K)")
    T, K = x.shape
    E, N = w1.shape[0], w1.shape[1]
    pack = 2 if fmt == "mxfp4" else 1
    if N % 2:
        raise ValueError(f"N = {N} must be even (gate and up halves)")
    want = {"w1": (E, N, K // pack), "w2": (E, K, N // 2 // pack), "out": (T, K)}
    for name, t in (("w1", w1), ("w2", w2), ("out", out)):
        if tuple(t.shape) != want[name]:
            raise ValueError(f"{name} must have shape {want[name]}, got {tuple(t.shape)}")
    if topk_weights.dim() != 2 or topk_weights.shape[0] != T:
        raise ValueError(f"topk_weights must be (T={T}, top_k), got {tuple(topk_weights.shape)}")
    if expert_ids.numel() < (sorted_token_ids.numel() + block_m - 1) // block_m or num_tokens_post_padded.numel() < 1:
        raise ValueError("expert_ids must hold ceil(sorted_token_ids.numel() / block_m) entries and "
                         "num_tokens_post_padded one")
    tensors = [w1, w2, out, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded]
    if fmt != "bf16":
        if tuple(x_scales.shape) != (T, K // 32):
            raise ValueError(f"x_scales must have shape {(T, K // 32)}, got {tuple(x_scales.shape)}")
        for name, t, mn, ks in (("w1_scales_blocked", w1_scales, N, K // 32),
                                ("w2_scales_blocked", w2_scales, K, N // 2 // 32)):
            need = pack_scales_blocked_bytes(E, mn, ks)
            if t.numel() < need:
                raise ValueError(f"{name} must hold {need} bytes (pack_scales_blocked of ({E}, {mn}, {ks}))")
        tensors += [x_scales, w1_scales, w2_scales]
    for t in tensors:
        if t.device != x.device:
            raise ValueError(f"all tensors must be on {x.device}, got one on {t.device}")


def _same_device(first, *rest):
    for t in rest:
        if t.device != first.device:
            raise ValueError(f"all tensors must be on {first.device}, got one on {t.device}")


# ---------------------------------------------------------------- sizes
def moe_align_capacity(T: int, top_k: int, E: int, block_m: int) -> int:
    return int(load().moe_align_capacity(T, top_k, E, block_m))


def pack_scales_blocked_bytes(E: int, MN: int, KS: int) -> int:
    return int(load().pack_scales_blocked_bytes(E, MN, KS))


def moe_workspace_bytes(dtype: int, T: int, K: int, N: int, E: int, top_k: int, block_m: int) -> int:
    n = int(load().moe_workspace_bytes(dtype, T, K, N, E, top_k, block_m))
    if n < 0:
        raise MoeError(-1, "moe_workspace_bytes: invalid arguments")
    return n


# ---------------------------------------------------------------- calls
def moe_align(topk_ids, E: int, block_m: int, sorted_token_ids=None, expert_ids=None,
              num_tokens_post_padded=None, stream=None):
    """Routing planner.  Returns (sorted_token_ids, expert_ids, num_tokens_post_padded)."""
    import torch

    _need(topk_ids, "topk_ids", (torch.int32,))
    T, top_k = topk_ids.shape
    cap = moe_align_capacity(T, top_k, E, block_m)
    if cap < 0:
        raise MoeError(-1, "moe_align: invalid sizes")
    dev = topk_ids.device
    if sorted_token_ids is None:
        sorted_token_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    if expert_ids is None:
        expert_ids = torch.empty((sorted_token_ids.numel() + block_m - 1) // block_m, dtype=torch.int32,
                                 device=dev)
    if num_tokens_post_padded is None:
        num_tokens_post_padded = torch.empty(1, dtype=torch.int32, device=dev)
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    if expert_ids.numel() < (sorted_token_ids.numel() + block_m - 1) // block_m:
        raise ValueError("expert_ids must hold ceil(capacity / block_m) entries")
    _same_device(topk_ids, sorted_token_ids, expert_ids, num_tokens_post_padded)
    with _on_device(topk_ids.device, stream) as s:
        _check(load().moe_align(_ptr(topk_ids), T, top_k, E, block_m, _ptr(sorted_token_ids), _ptr(expert_ids),
                                _ptr(num_tokens_post_padded), sorted_token_ids.numel(), s))
    return sorted_token_ids, expert_ids, num_tokens_post_padded


def moe_route_align(logits, top_k: int, block_m: int, bias=None, topk_ids=None, topk_weights=None,
                    sorted_token_ids=None, expert_ids=None, num_tokens_post_padded=None, stream=None,
                    n_shared: int = 0):
    """Router + planner.  logits (T, E) fp32, bias (E,) fp32 or None; n_shared shared experts
    (indices E.., weight 1) follow the routed ones.  Returns (topk_ids, topk_weights,
    sorted_token_ids, expert_ids, num_tokens_post_padded), the first two (T, top_k + n_shared)."""
    import torch

    _need(logits, "logits", (torch.float32,))
    T, E = logits.shape
    if bias is not None:
        _need(bias, "bias", (torch.float32,))
        if bias.numel() != E:
            raise ValueError("bias must hold E values")
    kk = top_k + n_shared
    cap = moe_align_capacity(T, kk, E + n_shared, block_m)
    if cap < 0:
        raise MoeError(-1, "moe_route_align: invalid sizes")
    dev = logits.device
    if topk_ids is None:
        topk_ids = torch.empty((T, kk), dtype=torch.int32, device=dev)
    if topk_weights is None:
        topk_weights = torch.empty((T, kk), dtype=torch.float32, device=dev)
    if sorted_token_ids is None:
        sorted_token_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    if expert_ids is None:
        expert_ids = torch.empty((sorted_token_ids.numel() + block_m - 1) // block_m, dtype=torch.int32,
                                 device=dev)
    if num_tokens_post_padded is None:
        num_tokens_post_padded = torch.empty(1, dtype=torch.int32, device=dev)
    _need(topk_ids, "topk_ids", (torch.int32,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    if topk_ids.numel() < T * kk or topk_weights.numel() < T * kk:
        raise ValueError("topk_ids / topk_weights must hold T * (top_k + n_shared) entries")
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    if expert_ids.numel() < (sorted_token_ids.numel() + block_m - 1) // block_m:
        raise ValueError("expert_ids must hold ceil(capacity / block_m) entries")
    _same_device(logits, *([] if bias is None else [bias]), topk_ids, topk_weights, sorted_token_ids, expert_ids,
                 num_tokens_post_padded)
    with _on_device(logits.device, stream) as s:
        _check(load().moe_route_align(_ptr(logits), _ptr(bias), T, E, top_k, n_shared, block_m, _ptr(topk_ids),
                                      _ptr(topk_weights), _ptr(sorted_token_ids), _ptr(expert_ids),
                                      _ptr(num_tokens_post_padded), sorted_token_ids.numel(), s))
    return topk_ids, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded


def pack_scales_blocked(scales, out=None, stream=None):
    """(E, MN, KS) uint8 e8m0 scales, row major -> blocked 512-byte tiles (uint8, flat)."""
    import torch

    _need(scales, "scales", (torch.uint8,))
    E, MN, KS = scales.shape
    n = pack_scales_blocked_bytes(E, MN, KS)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=scales.device)
    _need(out, "out", (torch.uint8,))
    if out.numel() < n:
        raise ValueError(f"out must hold {n} bytes")
    _same_device(scales, out)
    with _on_device(scales.device, stream) as s:
        _check(load().pack_scales_blocked(_ptr(scales), _ptr(out), E, MN, KS, s))
    return out


def _workspace(dtype, T, K, N, E, top_k, block_m, workspace, device):
    import torch

    need = moe_workspace_bytes(dtype, T, K, N, E, top_k, block_m)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", (torch.uint8,))
    return workspace


def fused_moe_bf16(x, w1, w2, sorted_token_ids, expert_ids, num_tokens_post_padded, topk_weights, out,
                   block_m: int, workspace=None, tune: Tuning | None = None, stream=None):
    """bf16 path.  x (T,K), w1 (E,N,K), w2 (E,K,N/2) bf16; topk_weights (T,top_k) fp32; out (T,K) bf16."""
    import torch

    for t, n in ((x, "x"), (w1, "w1"), (w2, "w2"), (out, "out")):
        _need(t, n, (torch.bfloat16,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    _ffn_shapes("bf16", x, w1, w2, topk_weights, out, sorted_token_ids, expert_ids, num_tokens_post_padded, block_m)
    T, K = x.shape
    E, N, _ = w1.shape
    top_k = topk_weights.shape[1]
    ws = _workspace(DTYPE_BF16, T, K, N, E, top_k, block_m, workspace, x.device)
    _same_device(x, ws)
    with _on_device(x.device, stream) as s:
        _check(load().fused_moe_bf16(
            _ptr(x), _ptr(w1), _ptr(w2), _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded),
            _ptr(topk_weights), _ptr(out), T, K, N, E, top_k, block_m, sorted_token_ids.numel(), _ptr(ws),
            ws.numel(), None if tune is None else ctypes.byref(tune), s))
    return out


def fused_moe_mxfp8(x, x_scales, w1, w1_scales_blocked, w2, w2_scales_blocked, sorted_token_ids, expert_ids,
                    num_tokens_post_padded, topk_weights, out, block_m: int, workspace=None,
                    tune: Tuning | None = None, stream=None):
    """mxfp8 path.  e4m3 codes as uint8 (or float8_e4m3fn), e8m0 scales as uint8; out (T,K) bf16."""
    import torch

    u8 = (torch.uint8, torch.float8_e4m3fn)
    for t, n in ((x, "x"), (w1, "w1"), (w2, "w2")):
        _need(t, n, u8)
    for t, n in ((x_scales, "x_scales"), (w1_scales_blocked, "w1_scales_blocked"),
                 (w2_scales_blocked, "w2_scales_blocked")):
        _need(t, n, (torch.uint8,))
    _need(out, "out", (torch.bfloat16,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    _ffn_shapes("mxfp8", x, w1, w2, topk_weights, out, sorted_token_ids, expert_ids, num_tokens_post_padded, block_m,
                x_scales, w1_scales_blocked, w2_scales_blocked)
    T, K = x.shape
    E, N, _ = w1.shape
    top_k = topk_weights.shape[1]
    ws = _workspace(DTYPE_MXFP8, T, K, N, E, top_k, block_m, workspace, x.device)
    _same_device(x, ws)
    with _on_device(x.device, stream) as s:
        _check(load().fused_moe_mxfp8(
            _ptr(x), _ptr(x_scales), _ptr(w1), _ptr(w1_scales_blocked), _ptr(w2), _ptr(w2_scales_blocked),
            _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(topk_weights), _ptr(out),
            T, K, N, E, top_k, block_m, sorted_token_ids.numel(), _ptr(ws), ws.numel(),
            None if tune is None else ctypes.byref(tune), s))
    return out


def fused_moe_mxfp4(x, x_scales, w1, w1_scales_blocked, w2, w2_scales_blocked, sorted_token_ids, expert_ids,
                    num_tokens_post_padded, topk_weights, out, block_m: int, workspace=None,
                    tune: Tuning | None = None, stream=None):
    """mxfp8 activations, MXFP4 weights: w1 (E, N, K/2) and w2 (E, K, N/4) uint8 of packed e2m1 codes
    (even index in the low nibble); scales and the rest as fused_moe_mxfp8."""
    import torch

    _need(x, "x", (torch.uint8, torch.float8_e4m3fn))
    for t, n in ((w1, "w1"), (w2, "w2"), (x_scales, "x_scales"), (w1_scales_blocked, "w1_scales_blocked"),
                 (w2_scales_blocked, "w2_scales_blocked")):
        _need(t, n, (torch.uint8,))
    _need(out, "out", (torch.bfloat16,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    _ffn_shapes("mxfp4", x, w1, w2, topk_weights, out, sorted_token_ids, expert_ids, num_tokens_post_padded, block_m,
                x_scales, w1_scales_blocked, w2_scales_blocked)
    T, K = x.shape
    E, N, _ = w1.shape
    top_k = topk_weights.shape[1]
    ws = _workspace(DTYPE_MXFP4, T, K, N, E, top_k, block_m, workspace, x.device)
    _same_device(x, ws)
    with _on_device(x.device, stream) as s:
        _check(load().fused_moe_mxfp4(
            _ptr(x), _ptr(x_scales), _ptr(w1), _ptr(w1_scales_blocked), _ptr(w2), _ptr(w2_scales_blocked),
            _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(topk_weights), _ptr(out),
            T, K, N, E, top_k, block_m, sorted_token_ids.numel(), _ptr(ws), ws.numel(),
            None if tune is None else ctypes.byref(tune), s))
    return out


def fused_moe_bf16_noalloc_max_workspace() -> int:
    """Size of the library-owned workspace used by fused_moe_bf16_noalloc."""
    return int(load().fused_moe_bf16_noalloc_max_workspace())


def fused_moe_bf16_noalloc(x, w1, w2, sorted_token_ids, expert_ids, num_tokens_post_padded, topk_weights, out,
                           block_m: int, tune: Tuning | None = None, stream=None):
    """fused_moe_bf16 without a caller workspace: uses the library's fixed-size
    device scratch, so nothing is allocated.  For callers that cannot allocate
    device memory; problems needing more than
    fused_moe_bf16_noalloc_max_workspace() bytes are rejected."""
    import torch

    for t, n in ((x, "x"), (w1, "w1"), (w2, "w2"), (out, "out")):
        _need(t, n, (torch.bfloat16,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    for t, n in ((sorted_token_ids, "sorted_token_ids"), (expert_ids, "expert_ids"),
                 (num_tokens_post_padded, "num_tokens_post_padded")):
        _need(t, n, (torch.int32,))
    _ffn_shapes("bf16", x, w1, w2, topk_weights, out, sorted_token_ids, expert_ids, num_tokens_post_padded, block_m)
    T, K = x.shape
    E, N, _ = w1.shape
    top_k = topk_weights.shape[1]
    with _on_device(x.device, stream) as s:
        _check(load().fused_moe_bf16_noalloc(
            _ptr(x), _ptr(w1), _ptr(w2), _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded),
            _ptr(topk_weights), _ptr(out), T, K, N, E, top_k, block_m, sorted_token_ids.numel(),
            None if tune is None else ctypes.byref(tune), s))
    return out


def moe_ep_dispatch_plan(topk_ids, E: int, world: int, order=None, send_counts=None, stream=None):
    """Routes grouped by owner rank (experts split into `world` equal ranges).  Returns (order
    (T*top_k,) int32: route ids t*top_k+j reaching an expert, grouped by rank, then -1;
    send_counts (world,) int32)."""
    import torch

    _need(topk_ids, "topk_ids", (torch.int32,))
    T, top_k = topk_ids.shape
    dev = topk_ids.device
    order = torch.empty(T * top_k, dtype=torch.int32, device=dev) if order is None else order
    send_counts = torch.empty(world, dtype=torch.int32, device=dev) if send_counts is None else send_counts
    _need(order, "order", (torch.int32,))
    _need(send_counts, "send_counts", (torch.int32,))
    if order.numel() < T * top_k or send_counts.numel() < world:
        raise ValueError("order must hold T*top_k entries and send_counts world entries")
    _same_device(topk_ids, order, send_counts)
    with _on_device(dev, stream) as s:
        _check(load().moe_ep_dispatch_plan(_ptr(topk_ids), T, top_k, E, world, _ptr(order), _ptr(send_counts), s))
    return order, send_counts


def moe_ep_dispatch_pack(x, topk_ids, topk_weights, order, n: int, E: int, world: int, x_scales=None, stream=None):
    """The send buffers of the first n entries of `order`: (rows (n, K) in x's dtype, scales (n, K/32) uint8 or
    None, owner-local expert ids (n,) int32, routing weights (n,) fp32)."""
    import torch

    _need(topk_ids, "topk_ids", (torch.int32,))
    _need(topk_weights, "topk_weights", (torch.float32,))
    _need(order, "order", (torch.int32,))
    if not x.is_contiguous() or x.dim() != 2:
        raise ValueError("x must be a contiguous (T, K) tensor")
    T, top_k = topk_ids.shape
    if x.shape[0] != T or tuple(topk_weights.shape) != (T, top_k) or order.numel() < n:
        raise ValueError("x, topk_ids, topk_weights and order disagree in shape")
    dev = x.device
    rows = torch.empty((n, x.shape[1]), dtype=x.dtype, device=dev)
    scales = None
    if x_scales is not None:
        _need(x_scales, "x_scales", (torch.uint8,))
        if x_scales.shape[0] != T:
            raise ValueError("x_scales must have one row per token")
        scales = torch.empty((n, x_scales.shape[1]), dtype=torch.uint8, device=dev)
    local_e = torch.empty(n, dtype=torch.int32, device=dev)
    w = torch.empty(n, dtype=torch.float32, device=dev)
    _same_device(x, topk_ids, topk_weights, order, *([] if x_scales is None else [x_scales]))
    with _on_device(dev, stream) as s:
        _check(load().moe_ep_dispatch_pack(
            _ptr(x), x.shape[1] * x.element_size(), _ptr(x_scales), 0 if x_scales is None else x_scales.shape[1],
            _ptr(topk_ids), _ptr(topk_weights), _ptr(order), n, T, top_k, E, world, _ptr(rows), _ptr(scales),
            _ptr(local_e), _ptr(w), s))
    return rows, scales, local_e, w


def moe_ep_combine(y, order, n: int, T: int, top_k: int, out=None, slot=None, stream=None):
    """out (T, K) bf16: per token, the sum in route order (fp32) of its routes' rows of y (n, K) bf16, row i
    belonging to route order[i]."""
    import torch

    _need(y, "y", (torch.bfloat16,))
    _need(order, "order", (torch.int32,))
    K = y.shape[1]
    dev = y.device
    out = torch.empty((T, K), dtype=torch.bfloat16, device=dev) if out is None else out
    slot = torch.empty(max(T * top_k, 1), dtype=torch.int32, device=dev) if slot is None else slot
    _need(out, "out", (torch.bfloat16,))
    _need(slot, "slot", (torch.int32,))
    if tuple(out.shape) != (T, K) or slot.numel() < T * top_k or y.shape[0] < n or order.numel() < n:
        raise ValueError("out must be (T, K), slot hold T*top_k entries, y and order n rows")
    _same_device(y, order, out, slot)
    with _on_device(dev, stream) as s:
        _check(load().moe_ep_combine(_ptr(y), _ptr(order), n, T, top_k, K, _ptr(slot), _ptr(out), s))
    return out


def moe_device_status(stream=None, device=None):
    """Waits for the stream; raises MoeError(MOE_ERR_TIMEOUT) if a device-side wait of this library
    on that device gave up.  ``device``: default the stream's device, else the current one."""
    import torch

    if device is None:
        device = getattr(stream, "device", None) or torch.device("cuda", torch.cuda.current_device())
    with _on_device(torch.device(device), stream) as s:
        _check(load().moe_device_status(s))
