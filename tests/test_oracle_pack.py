"""Pins for the oracle's blocked weight-scale layout.

Source: "Prime Flash MoE: Fused MoE Kernels for Blackwell", Scale layout
(mxfp8): weight scales go into a sequence of 512-byte tiles, each covering a
128 MN x 128 K block.  Pinned by hand-worked byte positions (tests/golden),
the tile-size closed form, bijectivity on the valid region and the inverse."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_positions():
    E = MN = KS = None
    pos = []
    for line in open(os.path.join(GOLDEN, "pack_scales_positions.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *v = line.split()
        if key == "E":
            E = int(v[0])
        elif key == "MN":
            MN = int(v[0])
        elif key == "KS":
            KS = int(v[0])
        else:
            pos.append(tuple(int(a) for a in v))
    # value = 1 + a distinct id per (e, row, col), mod 255 (never 0)
    idx = np.arange(E * MN * KS).reshape(E, MN, KS)
    s = (idx % 251 + 1).astype(np.uint8)
    packed = oracle.pack_scales_blocked(s)
    assert packed.size == 4096
    for e, r, c, off in pos:
        assert packed[off] == s[e, r, c], (e, r, c, off)


@pytest.mark.parametrize("E,MN,KS", [(1, 128, 4), (2, 130, 5), (3, 256, 128), (2, 4096, 224), (1, 7, 1)])
def test_bijection_and_inverse(E, MN, KS):
    MT, KT = -(-MN // 128), -(-KS // 4)
    nbytes = E * MT * KT * 512
    idx = np.arange(E * MN * KS)
    # mark every valid entry with a unique 1-based id spread over two planes
    lo = (idx % 255 + 1).astype(np.uint8).reshape(E, MN, KS)
    hi = (idx // 255 % 255 + 1).astype(np.uint8).reshape(E, MN, KS)
    p_lo, p_hi = oracle.pack_scales_blocked(lo), oracle.pack_scales_blocked(hi)
    assert p_lo.size == nbytes
    filled = p_lo != 0
    assert filled.sum() == E * MN * KS                 # each valid entry lands once
    assert (p_hi[~filled] == 0).all()                  # pads are zero
    pairs = set(zip(p_lo[filled].tolist(), p_hi[filled].tolist()))
    assert len(pairs) == min(E * MN * KS, 255 * 255)
    assert np.array_equal(oracle.unpack_scales_blocked(p_lo, E, MN, KS), lo)


def test_tile_is_row_major_in_32_row_groups():
    # inside one tile, the 16-byte line l holds rows l, l+32, l+64, l+96 (4 bytes each)
    s = np.zeros((1, 128, 4), np.uint8)
    s[0, :, :] = (np.arange(128)[:, None] + 1).astype(np.uint8)
    t = oracle.pack_scales_blocked(s).reshape(32, 4, 4)   # (line, row-group, col)
    for line in range(32):
        for g in range(4):
            assert (t[line, g] == line + 32 * g + 1).all()
