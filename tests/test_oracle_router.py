"""Pins for the oracle's router (softmax -> top-k -> renormalise ahead of the planner).

Sources: "Prime Flash MoE: Fused MoE Kernels for Blackwell", Usage (topk_ids come from the
caller's gate) and "[RFC] Fused W8A8 MoE megakernel on H20", Results so far (both paths use
the same normalized routing weights).  Pinned by: hand-worked cases (tests/golden), torch's
float64 full softmax followed by gather-and-renormalise with torch.topk's selection on
tie-free inputs, top_k = E equal to the whole softmax, and invariants (weights sum to one,
descend with the scores, shift invariance on exactly representable scores, ties to the
lower index, top-1 weight exactly one).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "router_worked_example.txt")


def _val(tok: str) -> float:
    named = {"ln3": math.log(3.0), "ln2": math.log(2.0)}
    return named[tok] if tok in named else float(tok)


def _cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        if f[0] == "case":
            cur = {"name": f[1], "E": int(f[3]), "k": int(f[5])}
            cases.append(cur)
        elif f[0] == "logits":
            cur["logits"] = np.array([[_val(x) for x in f[1:]]], np.float32)
        elif f[0] == "bias":
            cur["bias"] = None if f[1] == "none" else np.array([_val(x) for x in f[1:]], np.float32)
        elif f[0] == "ids":
            cur["ids"] = [int(x) for x in f[1:]]
        elif f[0] == "weights":
            cur["weights"] = [float(x) for x in f[1:]]
    return cases


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_worked_examples(case):
    ids, w = oracle.route_topk(case["logits"], case["k"], case["bias"])
    assert ids[0].tolist() == case["ids"]
    np.testing.assert_allclose(w[0], case["weights"], rtol=0, atol=1e-7)


def test_against_torch_full_softmax():
    rng = np.random.default_rng(7)
    T, E, k = 96, 128, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = (-1.2 * np.log(rng.permutation(E) + 1.0)).astype(np.float32)
    ids, w = oracle.route_topk(logits, k, bias)
    z = torch.from_numpy(logits) + torch.from_numpy(bias)          # fp32 scores, one addition
    p = torch.softmax(z.double(), dim=1)                            # full softmax in float64
    top = torch.topk(z, k, dim=1)                                   # tie-free input: unique order
    assert np.array_equal(ids, top.indices.numpy().astype(np.int32))
    kept = torch.gather(p, 1, top.indices)
    ref = (kept / kept.sum(dim=1, keepdim=True)).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-12, atol=1e-15)


def test_top_k_equal_to_E_is_the_softmax():
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((5, 16)).astype(np.float32)
    ids, w = oracle.route_topk(logits, 16)
    p = torch.softmax(torch.from_numpy(logits).double(), dim=1).numpy()
    for t in range(5):
        assert sorted(ids[t].tolist()) == list(range(16))
        np.testing.assert_allclose(w[t], p[t, ids[t]], rtol=1e-12, atol=1e-15)
        assert np.all(np.diff(logits[t, ids[t]]) <= 0)


def test_invariants():
    rng = np.random.default_rng(9)
    # scores on a 1/64 grid in [-4, 4): adding 8 is exact in fp32, so the ranking is unchanged
    logits = (rng.integers(-256, 256, size=(40, 24)) / 64.0).astype(np.float32)
    ids, w = oracle.route_topk(logits, 6)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 1e-15)
    ids2, w2 = oracle.route_topk(logits + np.float32(8.0), 6)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(w, w2, rtol=1e-12)
    # ties go to the lower index: every equal run of scores appears in ascending expert order
    for t in range(40):
        for a, b in zip(ids[t][:-1], ids[t][1:]):
            if logits[t, a] == logits[t, b]:
                assert a < b


def test_top1_weight_is_one_and_bad_sizes_raise():
    ids, w = oracle.route_topk(np.array([[0.5, -1.0, 2.0]], np.float32), 1)
    assert ids.tolist() == [[2]] and w.tolist() == [[1.0]]
    with pytest.raises(RuntimeError):
        oracle.route_topk(np.zeros((2, 3), np.float32), 4)


def test_shared_experts_append_always_on_routes():
    rng = np.random.default_rng(10)
    logits = rng.standard_normal((12, 20)).astype(np.float32)
    ids0, w0 = oracle.route_topk(logits, 4)
    ids, w = oracle.route_topk(logits, 4, n_shared=2)
    assert ids.shape == (12, 6) and np.array_equal(ids[:, :4], ids0) and np.array_equal(w[:, :4], w0)
    assert (ids[:, 4] == 20).all() and (ids[:, 5] == 21).all() and (w[:, 4:] == 1.0).all()


def test_shared_expert_output_is_added_to_the_routed_sum():
    """A shared expert's contribution is its dense SwiGLU FFN with weight 1 (torch float64)."""
    import torch.nn.functional as F
    import workloads as W

    T, K, N, E, k = 10, 64, 128, 4, 2
    rng = np.random.default_rng(11)
    x = W.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    w1 = W.f32_to_bf16_bits((rng.standard_normal((E + 1, N, K)) / np.sqrt(K)).astype(np.float32))
    w2 = W.f32_to_bf16_bits((rng.standard_normal((E + 1, K, N // 2)) / np.sqrt(N // 2)).astype(np.float32))
    ids, w = oracle.route_topk(rng.standard_normal((T, E)).astype(np.float32), k, n_shared=1)
    both = oracle.fused_moe_bf16(x, w1, w2, ids, w.astype(np.float32), unrounded=True)[1]
    routed = oracle.fused_moe_bf16(x, w1, w2, ids[:, :k].copy(), w[:, :k].astype(np.float32), unrounded=True)[1]
    t = lambda b: torch.from_numpy(W.bf16_bits_to_f32(b)).double()
    h = F.linear(t(x), t(w1[E]))
    a = (F.silu(h[:, :N // 2]) * h[:, N // 2:]).to(torch.float32).to(torch.bfloat16).double()
    shared = F.linear(a, t(w2[E])).numpy()
    np.testing.assert_allclose(both, routed + shared, rtol=1e-12, atol=1e-12)
