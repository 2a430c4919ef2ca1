"""ep_forward with the library's kernels as the local forward, on one GPU: a one-rank NCCL group,
so dispatch and combine run through NCCL's all_to_all_single and every route lands on this rank.

Precision: the local forward returns every route's weighted output in bf16 (the fused kernels' output
type), and the combine sums those in fp32 -- one more bf16 rounding per route than the single-call
path.  The oracle emulates exactly that: each route alone (top-1 calls), rounded to bf16, summed in
order in float64.  Against it the bf16 path's tolerance applies.  Several ranks cannot be exercised
here: every GPU run has one GPU.
"""
import datetime
import socket

import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_bf16_parity, to_dev

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_single_rank_nccl():
    import torch
    import torch.distributed as dist
    from mixture_experts_ffn_planner_b200.ep import ep_forward, local_ffn_bf16

    sh = W.Shape(name="S", dtype="bf16", T=96, K=256, N=512, E=8, top_k=2, block_m=64, zipf_s=None)
    inp = W.inputs(sh, seed=21)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        x = to_dev(inp["x"], torch.bfloat16)
        w1, w2 = to_dev(inp["w1"], torch.bfloat16), to_dev(inp["w2"], torch.bfloat16)
        out = ep_forward(x, to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"]), sh.E,
                         local_ffn_bf16(w1, w2, sh.block_m))
        got = out.to(torch.bfloat16).view(torch.int16).cpu().numpy().astype(np.uint16)
    finally:
        dist.destroy_process_group()
    ref = np.zeros((sh.T, sh.K))
    for j in range(sh.top_k):      # each route's bf16-rounded output, summed in route order
        bits = oracle.fused_moe_bf16(inp["x"], inp["w1"], inp["w2"], inp["topk_ids"][:, j:j + 1].copy(),
                                     inp["topk_weights"][:, j:j + 1].copy())
        ref += W.bf16_bits_to_f32(bits).astype(np.float64)
    assert_bf16_parity(got, ref, "ep, one rank")
