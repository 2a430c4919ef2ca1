"""moe_align on the GPU against the oracle: bit-exact on every output word.

The planner is integer work (histogram, prefix sum over padded counts,
stable scatter of the flattened token*top_k+route ids), so every element of
sorted_token_ids, expert_ids and num_tokens_post_padded must equal the
oracle's, including the -1 padding and the -1 capacity tail.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


def _run(ids: np.ndarray, E: int, bm: int, cap: int | None = None):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    T, k = ids.shape
    need = moe.moe_align_capacity(T, k, E, bm)
    cap = need if cap is None else cap
    d_ids = to_dev(ids.astype(np.int32)) if ids.size else torch.empty((T, k), dtype=torch.int32, device="cuda")
    # poison the outputs so that any element the kernel skips shows up
    s = torch.full((cap,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    e = torch.full(((cap + bm - 1) // bm,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    moe.moe_align(d_ids, E, bm, s, e, n)
    torch.cuda.synchronize()
    return s.cpu().numpy(), e.cpu().numpy(), int(n.cpu().numpy()[0])


def _check(ids, E, bm, cap=None):
    T, k = ids.shape
    cap = oracle.align_capacity(T, k, E, bm) if cap is None else cap
    rs, re_, rn = oracle.moe_align(ids, E, bm, capacity=cap)
    gs, ge, gn = _run(ids, E, bm, cap)
    assert gn == rn
    np.testing.assert_array_equal(gs, rs)
    np.testing.assert_array_equal(ge, re_)


@pytest.mark.parametrize("bm", [16, 32, 64, 128])
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (7, 2, 4), (100, 3, 9), (333, 8, 64), (2048, 6, 256),
                                   (5000, 4, 1024), (4097, 8, 288),
                                   (12000, 4, 1024), (90000, 4, 1024)])  # the last: ids streamed, not staged
def test_random(T, k, E, bm):
    rng = np.random.default_rng(T * 131 + k * 7 + E + bm)
    ids = np.stack([rng.permutation(E)[:k] if k <= E else rng.integers(0, E, k) for _ in range(T)]).astype(np.int32)
    _check(ids, E, bm)


def test_duplicates_and_out_of_range_ids():
    rng = np.random.default_rng(5)
    ids = rng.integers(-3, 12, size=(257, 5)).astype(np.int32)  # ids < 0 or >= E route nowhere
    _check(ids, 10, 64)


@pytest.mark.parametrize("bm", [64, 128])
def test_edge_cases(bm):
    _check(np.zeros((0, 4), np.int32), 8, bm)                   # T = 0
    _check(np.full((1, 1), 3, np.int32), 8, bm)                 # one route
    _check(np.full((3000, 8), 5, np.int32), 16, bm)             # every route on one expert
    _check(np.full((5, 2), 1023, np.int32), 1024, bm)           # largest E, last expert only
    _check(np.arange(40, dtype=np.int32).reshape(20, 2) % 7, 7, bm)  # R < block_m per expert
    ids = np.random.default_rng(1).integers(0, 4, size=(50, 3)).astype(np.int32)
    _check(ids, 4, bm, cap=oracle.align_capacity(50, 3, 4, bm) + 517)  # spare capacity tail


@pytest.mark.parametrize("name", W.workload_names())
def test_workload_routing(name):
    """The planner on the routing of every workload at every token count."""
    for T in W.token_counts(name):
        sh = W.shape(name, T)
        ids, _ = W.routing(sh)
        _check(ids, sh.E, sh.block_m)


def test_large_R():
    """T*top_k = 65536 routes with Zipf-skewed routing (one expert takes most)."""
    sh = W.shape("C5", 8192)
    ids, _ = W.routing(sh)
    counts = np.bincount(ids.ravel(), minlength=sh.E)
    assert (counts == 0).any() and counts.max() > 4 * counts.mean()
    for bm in (64, 128):
        _check(ids, sh.E, bm)
