"""Shared helpers for the test suite: device transfer and the parity metrics.

The tolerances are the ones the fused MoE forward is specified against:
planner outputs bit-exact; bf16 path max|gpu - oracle| <= 2e-2 * rms(oracle);
mxfp8 path cosine >= 0.999 and max|gpu - oracle| <= 6e-2 * rms(oracle) -- the
difference of an element taken net of the GPU value's own rounding to bf16 (half
an ulp), since out is bf16 and the oracle value compared is its unrounded sum.
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


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |v| (8 significant bits): the most that rounding v to bf16 can move it."""
    a = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(np.maximum(a, 2.0 ** -126))        # a = m * 2^e, 0.5 <= m < 1
    return np.ldexp(1.0, e - 9)


def compare(gpu_bits: np.ndarray, ref: np.ndarray):
    """Returns (max arithmetic error / rms(ref), cosine, rms(ref), max|diff| / rms(ref)).

    ``ref`` is the oracle's out before its final bf16 rounding (float64).  out is bf16 ("Prime
    Flash MoE: Fused MoE Kernels for Blackwell", Shapes), so a correct GPU value differs from ref by
    its own rounding, up to half a bf16 ulp (2^-9 |out|: 2e-2 rms once |out| passes ~10 rms), on top
    of the arithmetic error the tolerance bounds; the arithmetic error of an element is therefore
    |diff| minus half an ulp of the GPU value (floored at 0).  bf16 bit patterns (uint16) are
    accepted for ref too."""
    g = bf16_bits_to_f64(gpu_bits).ravel()
    r = (bf16_bits_to_f64(ref) if ref.dtype == np.uint16 else np.asarray(ref, np.float64)).ravel()
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    d = np.abs(g - r)
    arith = np.maximum(d - bf16_half_ulp(g), 0.0)
    if rms == 0.0:
        m = float(np.max(d)) if g.size else 0.0
        return float(np.max(arith)) if g.size else 0.0, 1.0, 0.0, m
    rel = float(np.max(arith)) / rms
    den = float(np.linalg.norm(g) * np.linalg.norm(r))
    cos = float(np.dot(g, r) / den) if den > 0 else 0.0
    return rel, cos, rms, float(np.max(d)) / rms


def assert_bf16_parity(gpu_bits, ref_bits, what=""):
    rel, cos, rms, raw = compare(gpu_bits, ref_bits)
    assert rel <= BF16_MAX_REL, (f"{what}: max arithmetic error/rms = {rel:.3e} > {BF16_MAX_REL} (max|diff|/rms "
                                 f"{raw:.3e}, cos {cos:.6f}, rms {rms:.3e})")
    return rel, cos


def assert_mxfp8_parity(gpu_bits, ref_bits, what=""):
    rel, cos, rms, raw = compare(gpu_bits, ref_bits)
    assert cos >= MXFP8_MIN_COS and rel <= MXFP8_MAX_REL, \
        f"{what}: cos {cos:.6f} (>= {MXFP8_MIN_COS}), max arithmetic error/rms {rel:.3e} (<= {MXFP8_MAX_REL}; " \
        f"max|diff|/rms {raw:.3e}), rms {rms:.3e}"
    return rel, cos


def coverage_sample(sh, topk_ids: np.ndarray, n: int, seed: int = 20261202) -> np.ndarray:
    """A seeded sample of n tokens (all of them when n >= T) chosen to reach the places where a
    kernel fault would hide at full size:

    * a token of every non-empty expert while the sample has room (so every expert's weights,
      and with them every gate/up and down tile, enter the comparison), the most- and
      least-loaded experts first;
    * the tokens of the last row of every full block_m block, and of the first and last routed
      row of the last block, as the oracle's planner lays them out;
    * the rest drawn at random.
    """
    import oracle

    T = topk_ids.shape[0]
    if n >= T:
        return np.arange(T, dtype=np.int32)
    k = topk_ids.shape[1]
    flat = topk_ids.reshape(-1)
    valid = (flat >= 0) & (flat < sh.E)
    counts = np.bincount(flat[valid], minlength=sh.E)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 98, T, sh.E])))
    must = []
    seen = set()

    def add(t):
        t = int(t)
        if t not in seen:
            seen.add(t)
            must.append(t)

    sorted_ids, expert_ids, ntpp = oracle.moe_align(topk_ids, sh.E, sh.block_m)
    nblk = ntpp // sh.block_m
    blocks = sorted_ids[: nblk * sh.block_m].reshape(nblk, sh.block_m)
    last = blocks[:, -1]
    for r in last[last >= 0][: max(1, n // 8)]:          # last rows of full blocks
        add(r // k)
    if nblk:
        routed = blocks[-1][blocks[-1] >= 0]
        add(routed[0] // k)
        add(routed[-1] // k)
    order = np.argsort(-counts, kind="stable")
    used = [e for e in order if counts[e] > 0]
    first = [used[0], used[-1]] + [e for e in rng.permutation(used).tolist() if e not in (used[0], used[-1])]
    for e in first:                                       # one token per expert
        if len(must) >= n:
            break
        rows = np.nonzero((topk_ids == e).any(axis=1))[0]
        add(rows[rng.integers(len(rows))])
    must = must[:n]
    rest = [t for t in rng.permutation(T).tolist() if t not in seen]
    return np.array(sorted(must + rest[: max(0, n - len(must))]), dtype=np.int32)
