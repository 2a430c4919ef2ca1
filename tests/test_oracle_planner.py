"""Pins for the oracle planner (moe_align).

Definition: "[RFC] Fused W8A8 MoE megakernel on H20", Design (expert
histogram, prefix sums, row-to-token mapping); "Prime Flash MoE: Fused MoE
Kernels for Blackwell", API and Shapes (flattened token*top_k+route ids
grouped by expert, each group padded to block_m with -1, expert_ids per
block, num_tokens_post_padded).

Pinned by: a hand-worked example (tests/golden), an exhaustive comparison on
tiny inputs with a sort-based construction of the same output, and the
invariants that characterise the output completely."""
import itertools
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(path):
    kv = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        kv[key] = [int(v) for v in vals]
    return kv


def test_worked_example():
    kv = _read_kv(os.path.join(GOLDEN, "planner_worked_example.txt"))
    T, k, E, bm = kv["T"][0], kv["top_k"][0], kv["E"][0], kv["block_m"][0]
    ids = np.array(kv["topk_ids"], np.int32).reshape(T, k)
    s, e, n = oracle.moe_align(ids, E, bm)
    assert n == kv["num_tokens_post_padded"][0]
    assert s.tolist() == kv["sorted_token_ids"]
    assert e.tolist() == kv["expert_ids"]


def sort_based(ids, E, bm):
    """Independent construction: sort (expert, flattened id) pairs, then cut
    the sorted list into groups and pad each group to a block_m multiple."""
    flat = ids.reshape(-1).tolist()
    pairs = sorted((e, i) for i, e in enumerate(flat) if 0 <= e < E)
    out, blocks = [], []
    for e, grp in itertools.groupby(pairs, key=lambda p: p[0]):
        members = [i for _, i in grp]
        n_blk = -(-len(members) // bm)
        out += members + [-1] * (n_blk * bm - len(members))
        blocks += [e] * n_blk
    return out, blocks


@pytest.mark.parametrize("T,k,E,bm", [(2, 2, 3, 1), (2, 2, 3, 2), (3, 1, 4, 2), (1, 3, 3, 4), (2, 2, 2, 3)])
def test_exhaustive_tiny(T, k, E, bm):
    cap = oracle.align_capacity(T, k, E, bm)
    for combo in itertools.product(range(E), repeat=T * k):
        ids = np.array(combo, np.int32).reshape(T, k)
        s, e, n = oracle.moe_align(ids, E, bm)
        want_s, want_b = sort_based(ids, E, bm)
        assert n == len(want_s)
        assert s.tolist() == want_s + [-1] * (cap - len(want_s))
        assert e.tolist() == want_b + [-1] * (len(e) - len(want_b))


def check_invariants(ids, E, bm, s, e, n):
    R = ids.size
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    assert counts.sum() == R
    assert n == int(sum(-(-c // bm) * bm for c in counts))
    assert n % bm == 0
    body = s[:n]
    # every route appears exactly once, nothing else but padding
    assert np.array_equal(np.sort(body[body >= 0]), np.arange(R))
    assert (s[n:] == -1).all()
    nb = n // bm
    assert (e[nb:] == -1).all()
    assert (np.diff(e[:nb]) >= 0).all()
    for b in range(nb):
        blk = body[b * bm:(b + 1) * bm]
        real = blk[blk >= 0]
        assert (flat[real] == e[b]).all()             # single-expert block
        # padding only at the tail of a group
        if (blk < 0).any():
            first_pad = int(np.argmax(blk < 0))
            assert (blk[first_pad:] == -1).all()
            assert b + 1 == nb or e[b + 1] != e[b]
    for ex in range(E):
        members = body[np.repeat(e[:nb], bm) == ex]
        members = members[members >= 0]
        assert members.size == counts[ex]
        assert (np.diff(members) > 0).all()           # stable, ascending


@pytest.mark.parametrize("T,k,E,bm,seed", [(64, 2, 8, 64, 0), (256, 6, 256, 128, 1), (8192, 8, 288, 128, 2),
                                           (1, 8, 128, 128, 3), (513, 7, 33, 16, 4)])
def test_invariants_random(T, k, E, bm, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    s, e, n = oracle.moe_align(ids, E, bm)
    check_invariants(ids, E, bm, s, e, n)


def test_edge_cases():
    # all routes on one expert
    ids = np.full((100, 1), 3, np.int32)
    s, e, n = oracle.moe_align(ids, 5, 64)
    assert n == 128 and e.tolist()[:2] == [3, 3] and s[:100].tolist() == list(range(100))
    check_invariants(ids, 5, 64, s, e, n)
    # R < block_m
    ids = np.array([[1, 0]], np.int32)
    s, e, n = oracle.moe_align(ids, 4, 128)
    assert n == 256 and s[0] == 1 and s[128] == 0 and e[:2].tolist() == [0, 1]
    # T = 1, top_k = 1
    s, e, n = oracle.moe_align(np.array([[0]], np.int32), 1, 128)
    assert n == 128 and s[0] == 0 and (s[1:] == -1).all() and e[0] == 0


def test_skewed_routing_invariants():
    import workloads as W
    sh = W.shape("C5", 8192)
    ids, _ = W.routing(sh)
    s, e, n = oracle.moe_align(ids, sh.E, sh.block_m)
    check_invariants(ids, sh.E, sh.block_m, s, e, n)
