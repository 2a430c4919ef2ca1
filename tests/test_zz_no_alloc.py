"""fused_moe_bf16_noalloc: the bf16 forward for callers that cannot allocate
device memory (a plain C host without its own allocator, or a runtime whose
memory pool owns the whole device).  It uses the library's fixed-size device
scratch instead of a caller workspace.

Checked through the C ABI against fused_moe_bf16 with a caller-allocated
workspace, on two calls in a row (the scratch keeps the previous call's
contents, which must not leak into the next result), within the bf16
tolerance the other tests use.  This file is collected last so that a run
that stops at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest

import workloads as W
from tests.helpers import assert_bf16_parity, out_bits, to_dev

pytestmark = pytest.mark.gpu


def _problem(sh, seed):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    inp = W.inputs(sh, seed=seed)
    ids, tw = to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"])
    x, w1, w2 = (to_dev(inp[n], torch.bfloat16) for n in ("x", "w1", "w2"))
    s_ids, e_ids, ntpp = moe.moe_align(ids, sh.E, sh.block_m)
    return x, w1, w2, s_ids, e_ids, ntpp, tw


@pytest.mark.parametrize("sh", [
    W.Shape(name="S", dtype="bf16", T=200, K=256, N=512, E=8, top_k=2, block_m=128),
    W.shape("C1", 64),
], ids=["small", "C1"])
def test_noalloc_matches_workspace_call(sh):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    need = moe.moe_workspace_bytes(moe.DTYPE_BF16, sh.T, sh.K, sh.N, sh.E, sh.top_k, sh.block_m)
    assert need <= moe.fused_moe_bf16_noalloc_max_workspace()
    x, w1, w2, s_ids, e_ids, ntpp, tw = _problem(sh, seed=21)
    ref = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
    moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, tw, ref, sh.block_m)
    ref_bits = out_bits(ref)
    for call in range(2):
        out = torch.full((sh.T, sh.K), float("nan"), dtype=torch.bfloat16, device="cuda")
        moe.fused_moe_bf16_noalloc(x, w1, w2, s_ids, e_ids, ntpp, tw, out, sh.block_m)
        moe.moe_device_status()
        got = out_bits(out)
        assert_bf16_parity(got, ref_bits, f"noalloc call {call}")


def test_noalloc_second_problem_after_first():
    """A different (smaller) problem right after a larger one: stale scratch
    contents from the first call must not affect the second."""
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    for sh, seed in ((W.Shape(name="S", dtype="bf16", T=300, K=384, N=256, E=16, top_k=4, block_m=64), 5),
                     (W.Shape(name="S", dtype="bf16", T=37, K=128, N=128, E=5, top_k=2, block_m=32), 6)):
        x, w1, w2, s_ids, e_ids, ntpp, tw = _problem(sh, seed)
        ref = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
        moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, tw, ref, sh.block_m)
        out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
        moe.fused_moe_bf16_noalloc(x, w1, w2, s_ids, e_ids, ntpp, tw, out, sh.block_m)
        moe.moe_device_status()
        assert_bf16_parity(out_bits(out), out_bits(ref), f"T={sh.T}")


def test_noalloc_rejects_oversized_problem():
    """A problem whose workspace exceeds the built-in scratch is refused before launch."""
    import mixture_experts_ffn_planner_b200 as moe

    lib = moe.load()
    sh = W.shape("C2", 256)
    need = moe.moe_workspace_bytes(moe.DTYPE_BF16, sh.T, sh.K, sh.N, sh.E, sh.top_k, sh.block_m)
    assert need > moe.fused_moe_bf16_noalloc_max_workspace()
    cap = moe.moe_align_capacity(sh.T, sh.top_k, sh.E, sh.block_m)
    p = 256
    rc = lib.fused_moe_bf16_noalloc(p, p, p, p, p, p, p, p, sh.T, sh.K, sh.N, sh.E, sh.top_k, sh.block_m, cap,
                                    None, None)
    assert rc == -4 and b"scratch" in lib.moe_last_error()
    assert np.isfinite(need)
