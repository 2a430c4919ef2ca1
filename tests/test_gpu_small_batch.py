"""The small-batch form of the bf16 forward against the oracle.

For few routed rows fused_moe_bf16 runs two weight-streaming kernels after the planner -- one warp
per (block, 8 intermediate columns) for gate/up + SwiGLU, one per (block, 16 output features) for the
down projection, both on warp-level bf16 MMAs fed straight from memory -- then the route-order
combine.  `moe_tuning.small_batch` forces it on (1) or off (-1); by default it is taken when
T * top_k <= 128.  Tolerance: the bf16 path's (max arithmetic error <= 2e-2 * rms of the oracle out,
tests/helpers.py).  The cases cover one route, blocks with more rows than one pass takes (16), block
sizes 16..128, two blocks of one expert, invalid routes and a token with none, Zipf-skewed routing
with empty experts, a shape outside the form (N/2 not a multiple of 256), and the default switch at
C1 and C5.
"""
import numpy as np
import pytest

import workloads as W
from tests.helpers import assert_bf16_parity, out_bits, to_dev
from tests.test_gpu_ffn import gpu_forward, oracle_forward, small

pytestmark = pytest.mark.gpu


def tune(mode: int):
    import mixture_experts_ffn_planner_b200 as moe

    return moe.Tuning(small_batch=mode)


CASES = [
    small("bf16", 1, 256, 512, 8, 1, 128),            # one token, one route
    small("bf16", 3, 512, 512, 4, 4, 16),             # every expert routed, 16-row blocks
    small("bf16", 40, 256, 1024, 4, 2, 64),           # ~20 rows per block: two passes (16 + rest)
    small("bf16", 64, 1024, 1024, 8, 2, 64),          # the C1 shape
    small("bf16", 150, 256, 512, 2, 1, 128),          # 150 rows on 2 experts: two blocks of one expert
    small("bf16", 8, 4096, 512, 128, 8, 128, zipf=1.1),  # C5 T=8 shape, Zipf skew, empty experts
    small("bf16", 5, 512, 768, 6, 3, 32),             # N/2 = 384: not a multiple of 256 (tensor path)
]


@pytest.mark.parametrize("sh", CASES, ids=lambda s: f"T{s.T}-K{s.K}-N{s.N}-E{s.E}-k{s.top_k}-bm{s.block_m}")
def test_small_batch_matches_oracle(sh):
    inp = W.inputs(sh, seed=31)
    ref = oracle_forward(sh, inp)
    got = gpu_forward(sh, inp, tune=tune(1))
    rel, cos = assert_bf16_parity(got, ref, "small batch")
    print(f"SMALL-BATCH T={sh.T} K={sh.K} N={sh.N} E={sh.E} k={sh.top_k} bm={sh.block_m}: rel {rel:.3e} cos {cos:.7f}")


def test_small_batch_invalid_routes_and_empty_token():
    """Routes outside [0, E) add nothing; a token with no valid route gets a zero row."""
    sh = small("bf16", 24, 512, 512, 6, 3, 32)
    inp = W.inputs(sh, seed=32)
    ids = inp["topk_ids"].copy()
    ids[::4, 1] = -1
    ids[7, :] = sh.E + 3
    ids[11, 2] = sh.E
    inp["topk_ids"] = ids
    got = gpu_forward(sh, inp, tune=tune(1))
    assert_bf16_parity(got, oracle_forward(sh, inp), "small batch, invalid routes")
    assert np.all((got[7] & 0x7FFF) == 0), "a token without routes must come out zero"


def test_small_batch_deterministic_and_close_to_the_tensor_path():
    sh = small("bf16", 48, 1024, 1024, 8, 2, 64)
    inp = W.inputs(sh, seed=33)
    a, b = gpu_forward(sh, inp, tune=tune(1), repeat=2)
    np.testing.assert_array_equal(a, b)
    t = gpu_forward(sh, inp, tune=tune(-1))
    ref = oracle_forward(sh, inp)
    assert_bf16_parity(a, ref, "small batch")
    assert_bf16_parity(t, ref, "tensor path")


@pytest.mark.parametrize("name,T", [("C1", 64), ("C5", 1), ("C5", 8)])
def test_tensor_path_at_small_batch_sizes(name, T):
    """The default now takes the small-batch form at these sizes; the tensor-core phases stay
    correct there when forced."""
    sh = W.shape(name, T)
    inp = W.inputs(sh)
    assert_bf16_parity(gpu_forward(sh, inp, tune=tune(-1)), oracle_forward(sh, inp), f"{name} T={T} tensor path")


def test_small_batch_phase_events_and_workspace():
    """The phase hook still records four events (gate/up, down, combine), and a caller workspace of
    moe_workspace_bytes serves the small-batch form."""
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    sh = W.shape("C5", 8)
    inp = W.inputs(sh)
    ids, tw = to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"])
    s_ids, e_ids, ntpp = moe.moe_align(ids, sh.E, sh.block_m)
    x, w1, w2 = (to_dev(inp[n], torch.bfloat16) for n in ("x", "w1", "w2"))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    t = moe.Tuning.with_events(ev)
    t.small_batch = 1
    nbytes = moe.moe_workspace_bytes(moe.DTYPE_BF16, sh.T, sh.K, sh.N, sh.E, sh.top_k, sh.block_m)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
    moe.fused_moe_bf16(x, w1, w2, s_ids, e_ids, ntpp, tw, out, sh.block_m, workspace=ws, tune=t)
    torch.cuda.synchronize()
    moe.moe_device_status()
    ms = [ev[0].elapsed_time(ev[i]) for i in (1, 2, 3)]
    assert 0 < ms[0] <= ms[1] <= ms[2] + 1e-6
    assert_bf16_parity(out_bits(out), oracle_forward(sh, inp), "C5 T=8 small batch via workspace")
