"""Pins for the oracle's expert FFN (bf16 and mxfp8 paths).

Definition: "[RFC] Fused W8A8 MoE megakernel on H20", Background (gate/up
GroupGEMM, SiLU x gate + requant, down GroupGEMM, top-k weighted reduction)
and "Prime Flash MoE: Fused MoE Kernels for Blackwell", intro (SwiGLU from the
accumulator; mxfp8 requant of the intermediate), Shapes (w1 (E, N, K),
w2 (E, K, N/2), out (T, K) bf16, topk_weights fp32).

The oracle is checked against torch float64 library routines (F.linear,
F.silu) on the cases that reduce to a dense SwiGLU FFN, against a weighted sum
of such dense results for several routes, and against properties (linearity
in the routing weights, zero experts, zero input)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W


def _bf16_to_t(b):
    return torch.from_numpy(W.bf16_bits_to_f32(b)).double()


def _t_to_bf16_bits(t):
    return t.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)


def dense_swiglu_bf16(x, w1, w2, round_intermediate=True):
    """torch float64: bf16-rounded SwiGLU intermediate, dense FFN for one expert."""
    I = w1.shape[0] // 2
    h = F.linear(x, w1)
    a = F.silu(h[:, :I]) * h[:, I:]
    if round_intermediate:
        a = a.to(torch.float32).to(torch.bfloat16).double()
    return F.linear(a, w2)


def _small_inputs(T, K, N, E, k, seed):
    rng = np.random.default_rng(seed)
    x = W.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    w1 = W.f32_to_bf16_bits((rng.standard_normal((E, N, K)) / np.sqrt(K)).astype(np.float32))
    w2 = W.f32_to_bf16_bits((rng.standard_normal((E, K, N // 2)) / np.sqrt(N // 2)).astype(np.float32))
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    tw = rng.random((T, k)).astype(np.float32) + 0.1
    tw /= tw.sum(axis=1, keepdims=True)
    return x, w1, w2, ids, tw.astype(np.float32)


@pytest.mark.parametrize("K,N", [(64, 96), (96, 64), (128, 256)])
def test_bf16_top1_is_dense_swiglu(K, N):
    T, E = 40, 3
    x, w1, w2, _, _ = _small_inputs(T, K, N, E, 1, seed=K + N)
    ids = (np.arange(T) % E).astype(np.int32)[:, None]
    tw = np.ones((T, 1), np.float32)
    out = oracle.fused_moe_bf16(x, w1, w2, ids, tw)
    xt = _bf16_to_t(x)
    for e in range(E):
        rows = np.nonzero(ids[:, 0] == e)[0]
        ref = dense_swiglu_bf16(xt[rows], _bf16_to_t(w1[e]), _bf16_to_t(w2[e]))
        ref_bits = _t_to_bf16_bits(ref)
        got = W.bf16_bits_to_f32(out[rows]).astype(np.float64)
        # same bf16 value except on rare rounding-order ties
        assert (out[rows] == ref_bits).mean() > 0.995
        assert np.abs(got - ref.numpy()).max() <= 2.0 ** -7 * np.abs(ref.numpy()).max()


def test_bf16_intermediate_rounding_is_visible():
    """The oracle rounds the SwiGLU intermediate to bf16: it agrees with the
    torch path that rounds it much more often than with the one that does not."""
    T, K, N, E = 64, 32, 512, 1
    x, w1, w2, _, _ = _small_inputs(T, K, N, E, 1, seed=7)
    ids = np.zeros((T, 1), np.int32)
    out = oracle.fused_moe_bf16(x, w1, w2, ids, np.ones((T, 1), np.float32))
    xt, a1, a2 = _bf16_to_t(x), _bf16_to_t(w1[0]), _bf16_to_t(w2[0])
    with_r = _t_to_bf16_bits(dense_swiglu_bf16(xt, a1, a2, True))
    without = _t_to_bf16_bits(dense_swiglu_bf16(xt, a1, a2, False))
    m_with, m_without = (out == with_r).mean(), (out == without).mean()
    assert m_with > 0.995 and m_without < m_with - 0.02, (m_with, m_without)


def test_bf16_topk_is_weighted_sum_of_dense_experts():
    T, K, N, E, k = 24, 64, 128, 5, 3
    x, w1, w2, ids, tw = _small_inputs(T, K, N, E, k, seed=11)
    out = W.bf16_bits_to_f32(oracle.fused_moe_bf16(x, w1, w2, ids, tw)).astype(np.float64)
    xt = _bf16_to_t(x)
    ref = np.zeros((T, K))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            y = dense_swiglu_bf16(xt[t:t + 1], _bf16_to_t(w1[e]), _bf16_to_t(w2[e]))[0].numpy()
            ref[t] += float(tw[t, j]) * y
    assert np.abs(out - ref).max() <= 2.0 ** -8 * np.abs(ref).max() * 1.01


def test_bf16_linear_in_routing_weights_and_zero_cases():
    T, K, N, E, k = 16, 64, 128, 4, 2
    x, w1, w2, ids, tw = _small_inputs(T, K, N, E, k, seed=3)
    base = oracle.fused_moe_bf16(x, w1, w2, ids, tw)
    # doubling every routing weight doubles the output exactly (powers of two)
    dbl = oracle.fused_moe_bf16(x, w1, w2, ids, (tw * 2).astype(np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(dbl), 2 * W.bf16_bits_to_f32(base))
    # a route with weight 0 contributes nothing
    tw0 = tw.copy()
    tw0[:, 1] = 0
    one = oracle.fused_moe_bf16(x, w1, w2, ids[:, :1].copy(), tw0[:, :1].copy())
    assert np.array_equal(oracle.fused_moe_bf16(x, w1, w2, ids, tw0), one)
    # an expert whose w2 is zero contributes nothing
    w2z = w2.copy()
    w2z[ids[:, 1]] = 0
    got = oracle.fused_moe_bf16(x, w1, w2z, ids, tw)
    w2only = w2.copy()
    w2only[ids[:, 1]] = 0
    assert np.array_equal(got, oracle.fused_moe_bf16(x, w1, w2only, ids, tw))
    # zero input gives exactly zero output
    assert not oracle.fused_moe_bf16(np.zeros_like(x), w1, w2, ids, tw).any()
    # the token subset reproduces the full rows
    sub = np.array([0, 5, 15], np.int32)
    part = oracle.fused_moe_bf16(x, w1, w2, ids, tw, tokens=sub)
    assert np.array_equal(part[sub], base[sub]) and not np.delete(part, sub, axis=0).any()


# --------------------------------------------------------------- mxfp8 ----
def _deq(codes, scales):
    """Library dequantisation: torch's float8 decode times 2^(s-127)."""
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double()
    s = torch.from_numpy(scales.astype(np.float64) - 127.0)
    return v * torch.exp2(s).repeat_interleave(32, dim=-1)


def _mx_inputs(T, K, N, E, seed):
    rng = np.random.default_rng(seed)
    xq, xs = W.mx_quantize_inputs(rng.standard_normal((T, K)).astype(np.float32))
    w1q, s1 = W.mx_quantize_inputs((rng.standard_normal((E, N, K)) / np.sqrt(K)).astype(np.float32))
    w2q, s2 = W.mx_quantize_inputs((rng.standard_normal((E, K, N // 2)) / np.sqrt(N // 2)).astype(np.float32))
    return xq, xs, w1q, s1, w2q, s2


@pytest.mark.parametrize("K,N", [(64, 128), (128, 64), (256, 512)])
def test_mxfp8_top1_is_dense_with_requant(K, N):
    T, E = 32, 2
    xq, xs, w1q, s1, w2q, s2 = _mx_inputs(T, K, N, E, seed=K * 3 + N)
    ids = (np.arange(T) % E).astype(np.int32)[:, None]
    out = oracle.fused_moe_mxfp8(xq, xs, w1q, s1, w2q, s2, ids, np.ones((T, 1), np.float32))
    I = N // 2
    xd = _deq(xq, xs)
    for e in range(E):
        rows = np.nonzero(ids[:, 0] == e)[0]
        h = F.linear(xd[rows], _deq(w1q[e], s1[e]))
        a32 = (F.silu(h[:, :I]) * h[:, I:]).to(torch.float32).numpy()
        aq, ascale = W.mx_quantize_inputs(a32)          # independent quantiser
        y = F.linear(_deq(aq, ascale), _deq(w2q[e], s2[e]))
        ref_bits = _t_to_bf16_bits(y)
        assert (out[rows] == ref_bits).mean() > 0.995
        got = W.bf16_bits_to_f32(out[rows]).astype(np.float64)
        assert np.abs(got - y.numpy()).max() <= 2.0 ** -7 * np.abs(y.numpy()).max()


def test_mxfp8_topk_weighted_and_zero():
    T, K, N, E, k = 12, 64, 128, 4, 2
    xq, xs, w1q, s1, w2q, s2 = _mx_inputs(T, K, N, E, seed=21)
    rng = np.random.default_rng(0)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    tw = np.full((T, k), 0.5, np.float32)
    both = W.bf16_bits_to_f32(oracle.fused_moe_mxfp8(xq, xs, w1q, s1, w2q, s2, ids, tw)).astype(np.float64)
    parts = 0
    for j in range(k):
        o = oracle.fused_moe_mxfp8(xq, xs, w1q, s1, w2q, s2, ids[:, j:j + 1].copy(),
                                   np.ones((T, 1), np.float32))
        parts = parts + 0.5 * W.bf16_bits_to_f32(o).astype(np.float64)
    assert np.abs(both - parts).max() <= 2.0 ** -7 * np.abs(parts).max()
    assert not oracle.fused_moe_mxfp8(np.zeros_like(xq), xs, w1q, s1, w2q, s2, ids, tw).any()


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_unrounded_output(dtype):
    """out_f64 is out before its last rounding: rounding it gives out exactly,
    and on the dense top-1 case it matches torch float64 to double precision
    (up to the bf16 / mxfp8 rounding of the intermediate, done identically)."""
    T, K, N, E = 24, 64, 128, 3
    x, w1, w2, ids, tw = _small_inputs(T, K, N, E, 2, seed=99)
    if dtype == "bf16":
        out, f64 = oracle.fused_moe_bf16(x, w1, w2, ids, tw, unrounded=True)
    else:
        xq, xs = W.mx_quantize_inputs(W.bf16_bits_to_f32(x))
        w1q, s1 = W.mx_quantize_inputs(W.bf16_bits_to_f32(w1))
        w2q, s2 = W.mx_quantize_inputs(W.bf16_bits_to_f32(w2))
        out, f64 = oracle.fused_moe_mxfp8(xq, xs, w1q, s1, w2q, s2, ids, tw, unrounded=True)
    again = np.array([oracle.double_to_bf16(v) for v in f64.ravel()], dtype=np.uint16).reshape(out.shape)
    np.testing.assert_array_equal(again, out)
    assert np.abs(f64 - W.bf16_bits_to_f32(out)).max() <= 2.0 ** -8 * np.abs(f64).max()
    # sampled rows, other rows untouched
    sub = np.array([1, 7, 20], np.int32)
    if dtype == "bf16":
        _, part = oracle.fused_moe_bf16(x, w1, w2, ids, tw, tokens=sub, unrounded=True)
    else:
        _, part = oracle.fused_moe_mxfp8(xq, xs, w1q, s1, w2q, s2, ids, tw, tokens=sub, unrounded=True)
    np.testing.assert_array_equal(part[sub], f64[sub])
    assert not np.delete(part, sub, axis=0).any()


def test_unrounded_dense_top1_matches_torch():
    T, K, N, E = 30, 96, 64, 2
    x, w1, w2, _, _ = _small_inputs(T, K, N, E, 1, seed=5)
    ids = (np.arange(T) % E).astype(np.int32)[:, None]
    _, f64 = oracle.fused_moe_bf16(x, w1, w2, ids, np.ones((T, 1), np.float32), unrounded=True)
    xt = _bf16_to_t(x)
    for e in range(E):
        rows = np.nonzero(ids[:, 0] == e)[0]
        h = F.linear(xt[rows], _bf16_to_t(w1[e]))
        a = F.silu(h[:, : N // 2]) * h[:, N // 2:]
        a_bits = np.array([oracle.double_to_bf16(v) for v in a.numpy().ravel()], np.uint16).reshape(a.shape)
        ref = F.linear(torch.from_numpy(W.bf16_bits_to_f32(a_bits)).double(), _bf16_to_t(w2[e])).numpy()
        np.testing.assert_allclose(f64[rows], ref, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_final_rounding_is_one_rounding_of_the_exact_sum(dtype):
    """out = RNE_bf16 of the exact route sum, rounded once.

    The inputs make the intermediate exactly 1:
    - x = 8 in column 0;
    - the gate row is 8, so g = 64 and silu(64) = 64 to double precision;
    - the up row is 2^-9, so u = 1/64.
    With w2 = +-1, each route's result is +-1. The token's two routes carry weights 1 + 2^-8 and 2^-30,
    so the exact sum is 1 + 2^-8 + 2^-30. That lies just above the midpoint of the bf16 neighbours 1 and
    1 + 2^-7, so it rounds up to 0x3F81. Rounding through fp32 first would land on the midpoint itself
    and tie to even (0x3F80)."""
    K, E = 32, 1
    N = 4 if dtype == "bf16" else 64          # the mxfp8 path needs N/2 to be a multiple of 32
    I = N // 2
    ids = np.zeros((1, 2), np.int32)          # both routes to expert 0
    tw = np.array([[1.0 + 2.0 ** -8, 2.0 ** -30]], np.float32)
    assert float(tw[0, 0]) + float(tw[0, 1]) == 1.0 + 2.0 ** -8 + 2.0 ** -30
    if dtype == "bf16":
        bf = {8.0: 0x4100, 2.0 ** -9: 0x3B00, 1.0: 0x3F80, -1.0: 0xBF80}
        x = np.zeros((1, K), np.uint16)
        x[0, 0] = bf[8.0]
        w1 = np.zeros((E, N, K), np.uint16)
        w1[0, 0, 0], w1[0, I, 0] = bf[8.0], bf[2.0 ** -9]
        w2 = np.zeros((E, K, I), np.uint16)
        w2[0, 0, 0], w2[0, 1, 0] = bf[1.0], bf[-1.0]
        out, f64 = oracle.fused_moe_bf16(x, w1, w2, ids, tw, unrounded=True)
    else:
        # e4m3 codes: 8.0 = 0x50, 1.0 = 0x38, -1.0 = 0xB8; e8m0 byte 127 = 2^0, 118 = 2^-9
        x = np.zeros((1, K), np.uint8)
        x[0, 0] = 0x50
        xs = np.full((1, K // 32), 127, np.uint8)
        w1 = np.zeros((E, N, K), np.uint8)
        w1[0, 0, 0], w1[0, I, 0] = 0x50, 0x38
        s1 = np.full((E, N, K // 32), 127, np.uint8)
        s1[0, I, 0] = 118
        w2 = np.zeros((E, K, I), np.uint8)
        w2[0, 0, 0], w2[0, 1, 0] = 0x38, 0xB8
        s2 = np.full((E, K, I // 32), 127, np.uint8)
        out, f64 = oracle.fused_moe_mxfp8(x, xs, w1, s1, w2, s2, ids, tw, unrounded=True)
    assert f64[0, 0] == 1.0 + 2.0 ** -8 + 2.0 ** -30 and f64[0, 1] == -f64[0, 0]
    assert int(out[0, 0]) == 0x3F81 and int(out[0, 1]) == 0xBF81
    assert not f64[0, 2:].any() and not out[0, 2:].any()
