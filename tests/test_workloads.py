"""Seeded input generators: determinism and the routing recipe's properties."""
import numpy as np

import workloads as W


def test_routing_properties():
    for name in W.workload_names():
        sh = W.shape(name, W.token_counts(name)[0])
        ids, tw = W.routing(sh)
        assert ids.shape == (sh.T, sh.top_k) and ids.dtype == np.int32
        assert ((ids >= 0) & (ids < sh.E)).all()
        assert all(len(set(r)) == sh.top_k for r in ids.tolist())       # distinct experts per token
        assert np.allclose(tw.sum(axis=1), 1.0, atol=1e-6)
        assert (np.diff(tw, axis=1) <= 0).all()                          # descending probability


def test_determinism_and_seed_dependence():
    sh = W.shape("C1", 64)
    a, b = W.bf16_inputs(sh), W.bf16_inputs(sh)
    for key in a:
        assert np.array_equal(a[key], b[key])
    c = W.bf16_inputs(sh, seed=1)
    assert not np.array_equal(a["w1"], c["w1"])


def test_zipf_skew_leaves_experts_empty():
    sh = W.shape("C5", 8)
    ids, _ = W.routing(sh)
    counts = np.bincount(ids.reshape(-1), minlength=sh.E)
    assert (counts == 0).sum() > sh.E // 2


def test_weight_scale():
    sh = W.shape("C1", 64)
    w = W.expert_f32(sh, "w1", 0)
    assert abs(w.std() * np.sqrt(sh.K) - 1.0) < 0.01


def test_sample_tokens_covers_extremes():
    sh = W.shape("C5", 512)
    ids, _ = W.routing(sh)
    tok = W.sample_tokens(sh, ids, 32)
    counts = np.bincount(ids.reshape(-1), minlength=sh.E)
    used = np.nonzero(counts)[0]
    hi, lo = used[np.argmax(counts[used])], used[np.argmin(counts[used])]
    assert (ids[tok] == hi).any() and (ids[tok] == lo).any()
    assert len(tok) == 32 and len(set(tok.tolist())) == 32
