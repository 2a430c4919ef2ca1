"""Pins for the oracle's MXFP4-weight path (mxfp8 activations x MXFP4 weights).

Element format: OCP MX v1.0 FP4 (E2M1): sign, 2 exponent bits (bias 1), 1 mantissa bit,
magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; one e8m0 scale per 32 values along the contraction
dimension.  The activation/weight pairing is the one of DeepGEMM #411 "SM90 FP8 x MXFP4
MegaMoE"; the forward is otherwise the mxfp8 path's ("Prime Flash MoE", intro: mxfp8 requant
of the intermediate).  Pinned by: the E2M1 code table, the caller-side quantiser's rounding
at every midpoint, torch float64 library routines on the dense top-1 case (weights
dequantised in the test with numpy bit operations, which fixes the nibble order), and
exact equality with the mxfp8 path when every weight is a value both formats hold.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W

# OCP E2M1, codes 0..7; codes 8..15 are their negatives
SPEC = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_code_table():
    for c in range(16):
        v = oracle.e2m1_to_double(c)
        want = SPEC[c & 7] * (-1.0 if c & 8 else 1.0)
        assert v == want and np.signbit(v) == bool(c & 8)


def test_quantiser_midpoints_ties_and_saturation():
    # a block with amax in [4, 8) has scale 2^0, so values are quantised as written
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.25, -0.75, 0.0, 6.0, 0.5, 1.0, -6.0, 4.0]
    want = [0, 2, 2, 4, 4, 6, 6, 7, 8, 10, 0, 7, 1, 2, 15, 6]   # ties to the even code; 7 saturates
    v = np.array([vals + [0.0] * 16], np.float32)
    packed, scales = W.mx_quantize_fp4(v)
    codes = np.stack([packed & 15, packed >> 4], axis=-1).reshape(1, -1)[0, :16]
    assert codes.tolist() == want and scales.tolist() == [[127]]
    # scale rule: floor(log2 amax) - 2
    for amax, byte in ((1.0, 125), (7.9, 127), (8.0, 128), (0.01, 118)):
        _, s = W.mx_quantize_fp4(np.array([[amax] + [0.0] * 31], np.float32))
        assert s[0, 0] == byte


def _deq_fp4(packed, scales):
    """Test-side dequantisation: low nibble = even index, magnitude table, sign bit, 2^(s-127)."""
    p = np.ascontiguousarray(packed)
    codes = np.stack([p & 15, p >> 4], axis=-1).reshape(p.shape[:-1] + (p.shape[-1] * 2,))
    mag = np.array(SPEC)[codes & 7]
    v = np.where(codes & 8, -mag, mag)
    return torch.from_numpy(v * np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=-1))


def _deq_fp8(codes, scales):
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double()
    return v * torch.exp2(torch.from_numpy(scales.astype(np.float64) - 127.0)).repeat_interleave(32, dim=-1)


def _inputs(T, K, N, E, seed):
    rng = np.random.default_rng(seed)
    xq, xs = W.mx_quantize_inputs(rng.standard_normal((T, K)).astype(np.float32))
    w1q, s1 = W.mx_quantize_fp4((rng.standard_normal((E, N, K)) / np.sqrt(K)).astype(np.float32))
    w2q, s2 = W.mx_quantize_fp4((rng.standard_normal((E, K, N // 2)) / np.sqrt(N // 2)).astype(np.float32))
    return xq, xs, w1q, s1, w2q, s2


@pytest.mark.parametrize("K,N", [(64, 128), (128, 64), (256, 512)])
def test_top1_is_dense_with_requant(K, N):
    T, E = 32, 2
    xq, xs, w1q, s1, w2q, s2 = _inputs(T, K, N, E, seed=K * 5 + N)
    ids = (np.arange(T) % E).astype(np.int32)[:, None]
    out = oracle.fused_moe_mxfp4(xq, xs, w1q, s1, w2q, s2, ids, np.ones((T, 1), np.float32))
    I = N // 2
    xd = _deq_fp8(xq, xs)
    for e in range(E):
        rows = np.nonzero(ids[:, 0] == e)[0]
        h = F.linear(xd[rows], _deq_fp4(w1q[e], s1[e]))
        a32 = (F.silu(h[:, :I]) * h[:, I:]).to(torch.float32).numpy()
        aq, ascale = W.mx_quantize_inputs(a32)
        y = F.linear(_deq_fp8(aq, ascale), _deq_fp4(w2q[e], s2[e]))
        got = W.bf16_bits_to_f32(out[rows]).astype(np.float64)
        assert np.abs(got - y.numpy()).max() <= 2.0 ** -7 * np.abs(y.numpy()).max()


def test_equals_mxfp8_path_on_shared_values():
    """Weights drawn from the E2M1 values times a power of two are exact in e4m3 too: the two
    paths must then agree bit for bit (same forward, different weight encodings)."""
    T, K, N, E, k = 16, 64, 128, 3, 2
    rng = np.random.default_rng(3)
    xq, xs = W.mx_quantize_inputs(rng.standard_normal((T, K)).astype(np.float32))

    def both(rows, cols):
        codes = rng.integers(0, 16, size=(E, rows, cols)).astype(np.uint8)
        codes[..., 0] = 7                                    # every block holds a 6: same amax
        mag = np.array(SPEC, np.float32)[codes & 7]
        v = np.where(codes & 8, -mag, mag).astype(np.float32) * np.float32(0.125)
        return W.mx_quantize_fp4(v), W.mx_quantize_inputs(v)
    (w1f, s1f), (w1e, s1e) = both(N, K)
    (w2f, s2f), (w2e, s2e) = both(K, N // 2)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    tw = np.full((T, k), 0.5, np.float32)
    a = oracle.fused_moe_mxfp4(xq, xs, w1f, s1f, w2f, s2f, ids, tw, unrounded=True)[1]
    b = oracle.fused_moe_mxfp8(xq, xs, w1e, s1e, w2e, s2e, ids, tw, unrounded=True)[1]
    assert np.array_equal(a, b)
