"""Pins for the oracle's scalar formats (bf16, OCP e4m3 / e8m0, the MX scale
rule) against closed forms and torch's own float8 / bfloat16 conversions.

Source of the formats: "Prime Flash MoE: Fused MoE Kernels for Blackwell",
intro table (bf16 / mxfp8 paths) and Scale layout (mxfp8) (block 32, OCP MX
quantiser, e8m0 scales)."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def _f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


# ---------------------------------------------------------------- e4m3 -----
def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_to_double(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])


def test_e4m3_closed_form():
    # largest finite, smallest normal, smallest subnormal, NaN codes
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x38) == 1.0
    assert oracle.e4m3_to_double(0xB8) == -1.0
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))


def test_e4m3_encode_roundtrip_every_finite_code():
    for c in range(256):
        v = oracle.e4m3_to_double(c)
        if math.isnan(v):
            continue
        assert oracle.double_to_e4m3(v) == c, (c, v)


def test_e4m3_encode_midpoints_ties_to_even_and_matches_torch():
    pos = sorted({oracle.e4m3_to_double(c) for c in range(0x7F)})  # 0 .. 448
    mids = [(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])]
    for m in mids:
        got = oracle.double_to_e4m3(m)
        lo = oracle.double_to_e4m3(max(v for v in pos if v < m))
        hi = oracle.double_to_e4m3(min(v for v in pos if v > m))
        assert got in (lo, hi)
        assert got % 2 == 0, (m, got)          # even mantissa wins a tie
        tref = torch.tensor([m], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item()
        assert got == tref, (m, got, tref)
        # just off the tie goes to the nearer neighbour
        eps = (oracle.e4m3_to_double(hi) - oracle.e4m3_to_double(lo)) * 1e-3
        assert oracle.double_to_e4m3(m - eps) == lo
        assert oracle.double_to_e4m3(m + eps) == hi
        assert oracle.double_to_e4m3(-m) == got | 0x80


def test_e4m3_saturates():
    for v in (448.0, 449.0, 463.99, 464.0, 479.0, 480.0, 1e6, 1e30):
        assert oracle.double_to_e4m3(v) == 0x7E
        assert oracle.double_to_e4m3(-v) == 0xFE
    assert oracle.double_to_e4m3(2.0 ** -11) == 0x00      # below half the smallest subnormal
    assert oracle.double_to_e4m3(3 * 2.0 ** -11) == 0x01  # 0.75 of it rounds up


# ---------------------------------------------------------------- e8m0 -----
def test_e8m0_decode():
    for c in range(255):
        assert oracle.e8m0_to_double(c) == 2.0 ** (c - 127)
    assert math.isnan(oracle.e8m0_to_double(255))


def test_mx_scale_rule_sweep():
    # amax = f * 2^p with 1 <= f < 2, so floor(log2 amax) = p; scale = 2^(p - 8)
    for p in range(-149, 128):
        for f in (1.0, 1.25, 1.5, 1.999):
            amax = f * 2.0 ** p
            if amax >= 2.0 ** 128 or _f32(amax) != amax:
                continue
            want = min(max(p - 8, -127), 127) + 127
            assert oracle.mx_scale_byte(amax) == want, (p, f)
    assert oracle.mx_scale_byte(0.0) == 0


def test_mx_quantize_hand_block():
    # one block: amax = 3.75 -> floor(log2 3.75) = 1 -> scale 2^(1-8) (byte 120)
    v = np.zeros(32, np.float32)
    v[0], v[1], v[2], v[3] = 3.75, -1.0, 0.001, 3.0
    codes, scales = oracle.mx_quantize(v)
    assert scales[0] == 120
    assert codes[0] == 0x7E                                  # 3.75 * 2^7 = 480 saturates to 448
    assert oracle.e4m3_to_double(codes[1]) == -128.0
    assert codes[2] == oracle.double_to_e4m3(0.001 * 128)
    assert oracle.e4m3_to_double(codes[3]) == 384.0          # 3 * 2^7
    z_codes, z_scales = oracle.mx_quantize(np.zeros(32, np.float32))
    assert z_scales[0] == 0 and not z_codes.any()


def test_mx_quantize_matches_caller_quantiser():
    """The oracle's requant routine (C) and the caller-side input quantiser
    (numpy + torch's float8 cast) are written independently; they must agree
    bit for bit over a wide dynamic range."""
    rng = np.random.default_rng(5)
    v = rng.standard_normal((64, 256)).astype(np.float32)
    v *= np.exp2(rng.integers(-30, 30, size=(64, 1))).astype(np.float32)
    v[3, :32] = 0.0
    v[4, 5] = 1e-40  # subnormal fp32 in an otherwise small block
    c1, s1 = oracle.mx_quantize(v)
    c2, s2 = W.mx_quantize_inputs(v)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)


# ---------------------------------------------------------------- bf16 -----
def test_bf16_roundtrip_and_torch():
    rng = np.random.default_rng(1)
    vals = rng.standard_normal(4000).astype(np.float32) * np.exp2(rng.integers(-130, 120, 4000)).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    for v, r in zip(vals.tolist(), ref.tolist()):
        assert oracle.double_to_bf16(v) == r, v
        back = torch.from_numpy(np.array([r], dtype=np.uint16).view(np.int16)).view(torch.bfloat16).double().item()
        assert oracle.bf16_to_double(r) == back


def test_bf16_ties_and_overflow():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties to 1 (even)
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is the midpoint of 1+2^-7 (odd) and 1+2^-6: ties up
    assert oracle.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.double_to_bf16(3.5e38) == 0x7F80 and oracle.double_to_bf16(-3.5e38) == 0xFF80
    assert oracle.double_to_bf16(2.0 ** -133) == 0x0001
    assert oracle.double_to_bf16(0.0) == 0 and oracle.double_to_bf16(-0.0) == 0x8000


def test_caller_bf16_conversion_matches_torch():
    rng = np.random.default_rng(2)
    v = rng.standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(W.f32_to_bf16_bits(v), ref)


@pytest.mark.parametrize("x", [1.0, -2.5, 1e-3, 65504.0])
def test_bf16_decode(x):
    b = oracle.double_to_bf16(x)
    assert abs(oracle.bf16_to_double(b) - x) <= abs(x) * 2.0 ** -8
