"""Shared helpers for the test suite: device transfer and the parity metrics.

The tolerances are the ones the fused MoE forward is specified against:
planner outputs bit-exact; bf16 path max|gpu - oracle| <= 2e-2 * rms(oracle);
mxfp8 path cosine >= 0.999 and max|gpu - oracle| <= 6e-2 * rms(oracle).
"""
from __future__ import annotations

import numpy as np

BF16_MAX_REL = 2e-2
MXFP8_MAX_REL = 6e-2
MXFP8_MIN_COS = 0.999


def to_dev(a: np.ndarray, dtype=None):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(
        np.float64)


def out_bits(t) -> np.ndarray:
    """A (T, K) bf16 CUDA tensor -> host uint16 bit patterns."""
    import torch

    return t.view(torch.uint16).cpu().numpy() if hasattr(torch, "uint16") else t.view(torch.int16).cpu().numpy().view(
        np.uint16)


def compare(gpu_bits: np.ndarray, ref: np.ndarray):
    """Returns (max|diff| / rms(ref), cosine, rms(ref)).

    ``ref`` is the oracle's out before its final bf16 rounding (float64); the
    last rounding is a decision the two sides take in different precision
    and may land one bf16 ulp apart, more than the tolerance at large |out|.
    bf16 bit patterns (uint16) are accepted too."""
    g = bf16_bits_to_f64(gpu_bits).ravel()
    r = (bf16_bits_to_f64(ref) if ref.dtype == np.uint16 else np.asarray(ref, np.float64)).ravel()
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    if rms == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0, 1.0, 0.0
    rel = float(np.max(np.abs(g - r))) / rms
    den = float(np.linalg.norm(g) * np.linalg.norm(r))
    cos = float(np.dot(g, r) / den) if den > 0 else 0.0
    return rel, cos, rms


def assert_bf16_parity(gpu_bits, ref_bits, what=""):
    rel, cos, rms = compare(gpu_bits, ref_bits)
    assert rel <= BF16_MAX_REL, f"{what}: max|diff|/rms = {rel:.3e} > {BF16_MAX_REL} (cos {cos:.6f}, rms {rms:.3e})"
    return rel, cos


def assert_mxfp8_parity(gpu_bits, ref_bits, what=""):
    rel, cos, rms = compare(gpu_bits, ref_bits)
    assert cos >= MXFP8_MIN_COS and rel <= MXFP8_MAX_REL, \
        f"{what}: cos {cos:.6f} (>= {MXFP8_MIN_COS}), max|diff|/rms {rel:.3e} (<= {MXFP8_MAX_REL}), rms {rms:.3e}"
    return rel, cos
