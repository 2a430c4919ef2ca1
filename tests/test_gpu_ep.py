"""Expert-parallel forward on one GPU: the dispatch/combine kernels against the plain torch reference
(tests/ep_reference_ops.py), and ep_forward with the library's kernels as a one-rank NCCL group, so
dispatch and combine run through NCCL's all_to_all_single and every route lands on this rank.

Plan and pack are integer and byte work: bit-exact against the reference for 1, 2, 4 and 8 ranks' worth
of experts (the kernels do not communicate, so the grouping for several ranks runs on one device).  The
combine sums bf16 rows in fp32 in route order and rounds once: bit-exact against the same sequential
fp32 sum in numpy.

Precision of ep_forward: the local forward returns every route's weighted output in bf16 (the fused
kernels' output type), and the combine sums those in fp32 -- one more bf16 rounding per route than the
single-call path.  The oracle emulates exactly that: each route alone (top-1 calls), rounded to bf16,
summed in order in float64.  Against it the path's tolerance applies (bf16, or mxfp8).  Several ranks
cannot be exercised here: every GPU run has one GPU.
"""
import datetime
import socket

import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_bf16_parity, assert_mxfp8_parity, out_bits, to_dev

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routes(T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32) if T else np.zeros((0, k), np.int32)
    if T > 3:
        ids[1, 0] = -1          # routes to nowhere
        ids[3, :] = E + 2       # a token with no valid route
    return ids, (rng.random((T, k)) + 0.1).astype(np.float32)


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("T", [0, 1, 37, 3000])
def test_dispatch_kernels_match_the_reference(world, T):
    import torch
    import mixture_experts_ffn_planner_b200 as moe
    from tests.ep_reference_ops import TorchOps

    E, k, K = 32, 4, 256
    ids, tw = _routes(T, k, E, seed=T + world)
    ids_d, tw_d = to_dev(ids), to_dev(tw)
    order, counts = moe.moe_ep_dispatch_plan(ids_d, E, world)
    r_order, r_counts = TorchOps().plan(torch.from_numpy(ids), E, world)
    np.testing.assert_array_equal(order.cpu().numpy(), r_order.numpy())
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts.numpy())
    n = int(r_counts.sum())
    rng = np.random.default_rng(7)
    x = rng.integers(0, 256, (T, K), dtype=np.uint8)
    xs = rng.integers(100, 140, (T, K // 32), dtype=np.uint8)
    got = moe.moe_ep_dispatch_pack(to_dev(x), ids_d, tw_d, order, n, E, world, x_scales=to_dev(xs))
    ref = TorchOps().pack(torch.from_numpy(x), torch.from_numpy(xs), torch.from_numpy(ids), torch.from_numpy(tw),
                          r_order, n, E, world)
    for g, r in zip(got, ref):
        np.testing.assert_array_equal(g.cpu().numpy(), r.numpy())


@pytest.mark.parametrize("T,k", [(1, 1), (50, 3), (2000, 8)])
def test_combine_kernel_is_the_route_order_fp32_sum(T, k):
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    E, K, world = 16, 512, 4
    ids, _ = _routes(T, k, E, seed=3 * T + k)
    order, counts = moe.moe_ep_dispatch_plan(to_dev(ids), E, world)
    n = int(counts.sum())
    rng = np.random.default_rng(11)
    y = W.f32_to_bf16_bits(rng.standard_normal((n, K)).astype(np.float32))
    out = moe.moe_ep_combine(to_dev(y, torch.bfloat16), order, n, T, k)
    o = order.cpu().numpy()[:n]
    slot = np.full(T * k, -1, np.int64)
    slot[o] = np.arange(n)
    yf = W.bf16_bits_to_f32(y)
    acc = np.zeros((T, K), np.float32)
    for j in range(k):
        s = slot.reshape(T, k)[:, j]
        acc += np.where(s[:, None] >= 0, yf[np.maximum(s, 0)], np.float32(0))
    np.testing.assert_array_equal(out_bits(out), W.f32_to_bf16_bits(acc))


def _nccl_one_rank():
    import torch
    import torch.distributed as dist

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))


def _route_by_route_oracle(sh, inp, fwd):
    """Each route alone through the oracle (top-1), rounded to bf16, summed in route order in float64."""
    ref = np.zeros((sh.T, sh.K))
    for j in range(sh.top_k):
        bits = fwd(inp["topk_ids"][:, j:j + 1].copy(), inp["topk_weights"][:, j:j + 1].copy())
        ref += W.bf16_bits_to_f32(bits).astype(np.float64)
    return ref


def test_ep_single_rank_nccl_bf16():
    import torch
    import torch.distributed as dist
    from mixture_experts_ffn_planner_b200.ep import ep_forward, local_ffn_bf16

    sh = W.Shape(name="S", dtype="bf16", T=96, K=256, N=512, E=8, top_k=2, block_m=64, zipf_s=None)
    inp = W.inputs(sh, seed=21)
    _nccl_one_rank()
    try:
        x = to_dev(inp["x"], torch.bfloat16)
        w1, w2 = to_dev(inp["w1"], torch.bfloat16), to_dev(inp["w2"], torch.bfloat16)
        out = ep_forward(x, to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"]), sh.E,
                         local_ffn_bf16(w1, w2, sh.block_m))
        got = out_bits(out)
    finally:
        dist.destroy_process_group()
    ref = _route_by_route_oracle(sh, inp, lambda ids, tw: oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], ids,
                                                                              tw))
    assert_bf16_parity(got, ref, "ep bf16, one rank")


def test_ep_single_rank_nccl_mxfp8():
    import torch
    import torch.distributed as dist
    import mixture_experts_ffn_planner_b200 as moe
    from mixture_experts_ffn_planner_b200.ep import ep_forward, local_ffn_mxfp8

    sh = W.Shape(name="S", dtype="mxfp8", T=96, K=512, N=512, E=8, top_k=3, block_m=64, zipf_s=None)
    inp = W.inputs(sh, seed=22)
    _nccl_one_rank()
    try:
        w1, w2 = to_dev(inp["w1"]), to_dev(inp["w2"])
        s1 = moe.pack_scales_blocked(to_dev(inp["w1_scales"]))
        s2 = moe.pack_scales_blocked(to_dev(inp["w2_scales"]))
        out = ep_forward(to_dev(inp["x"]), to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"]), sh.E,
                         local_ffn_mxfp8(w1, s1, w2, s2, sh.block_m), x_scales=to_dev(inp["x_scales"]))
        got = out_bits(out)
    finally:
        dist.destroy_process_group()
    ref = _route_by_route_oracle(sh, inp, lambda ids, tw: oracle.fused_moe_mxfp8(
        inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"], inp["w2_scales"], ids, tw))
    assert_mxfp8_parity(got, ref, "ep mxfp8, one rank")
