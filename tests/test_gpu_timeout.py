"""The bounded-wait path of the fused kernels, on the GPU, without a fault.

Every mbarrier wait in the fused kernels gives up after a limit (2 s by default); the kernel then
raises its CTA-wide abort flag, lets the copies it already issued land (bounded), frees its TMEM,
returns, and leaves MOE_ERR_TIMEOUT in the device status word.  Here the limit is set to 1 ns through
``moe_tuning.wait_timeout_ns``, so the first wait that does not succeed within one poll (an epilogue
warp waiting for a unit's accumulator, an MMA warp waiting for a TMA stage) runs out.  The test
checks that the call comes back, that moe_device_status reports the timeout once and then clears it,
and that the next call with the default limit on the same stream matches the oracle on a token
sample (the context is intact).
"""
import pytest

import oracle
import workloads as W
from tests.helpers import assert_bf16_parity, assert_mxfp8_parity, coverage_sample, out_bits, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
def test_wait_limit_runs_out_and_the_context_survives(dtype):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    # 2048 tokens x 2 routes over 8 experts: enough work units that no unit is split over K, so the
    # epilogue's wait for a unit's accumulator lasts the unit's whole K loop (K = 7168)
    sh = W.Shape(name="S", dtype=dtype, T=2048, K=7168, N=1024, E=8, top_k=2, block_m=128)
    inp = W.inputs(sh, seed=17)
    ids, tw = to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"])
    s_ids, e_ids, ntpp = moe.moe_align(ids, sh.E, sh.block_m)
    if dtype == "bf16":
        x, w1, w2 = (to_dev(inp[n], torch.bfloat16) for n in ("x", "w1", "w2"))

        def call(out, tune):
            moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, tw, out, sh.block_m, tune=tune)
    else:
        x, xs, w1, w2 = (to_dev(inp[n]) for n in ("x", "x_scales", "w1", "w2"))
        s1 = moe.pack_scales_blocked(to_dev(inp["w1_scales"]))
        s2 = moe.pack_scales_blocked(to_dev(inp["w2_scales"]))

        def call(out, tune):
            moe.fused_moe_mxfp8(x, xs, w1, s1, w2, s2, s_ids, e_ids, ntpp, tw, out, sh.block_m, tune=tune)

    moe.moe_device_status()  # nothing pending from earlier tests
    out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
    call(out, moe.Tuning(wait_timeout_ns=1))
    with pytest.raises(moe.MoeError) as err:
        moe.moe_device_status()
    assert err.value.code == -6 and err.value.name == "MOE_ERR_TIMEOUT"
    moe.moe_device_status()  # reported once, then cleared

    out = torch.full((sh.T, sh.K), float("nan"), dtype=torch.bfloat16, device="cuda")
    call(out, None)
    moe.moe_device_status()
    got = out_bits(out)
    toks = coverage_sample(sh, inp["topk_ids"], 192)
    if dtype == "bf16":
        ref = oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], inp["topk_ids"], inp["topk_weights"],
                                    tokens=toks, unrounded=True)[1]
        assert_bf16_parity(got[toks], ref[toks], "after a timed-out call")
    else:
        ref = oracle.fused_moe_mxfp8(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"],
                                     inp["w2_scales"], inp["topk_ids"], inp["topk_weights"], tokens=toks,
                                     unrounded=True)[1]
        assert_mxfp8_parity(got[toks], ref[toks], "after a timed-out call")
