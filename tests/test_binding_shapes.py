"""The binding's shape and device checks of the FFN calls (CPU).

The C ABI takes its sizes from x and w1 and trusts every other buffer. The binding therefore rejects
mismatched shapes before any launch. These checks look only at shapes and devices, so they run on CPU
tensors (and a `meta` tensor for the device check).
"""
import pytest
import torch

import mixture_experts_ffn_planner_b200 as moe

T, K, N, E, k, bm = 40, 256, 512, 4, 2, 64


def _args(fmt):
    pack = 2 if fmt == "mxfp4" else 1
    cap = moe.moe_align_capacity(T, k, E, bm)
    a = dict(x=torch.empty(T, K), w1=torch.empty(E, N, K // pack), w2=torch.empty(E, K, N // 2 // pack),
             topk_weights=torch.empty(T, k), out=torch.empty(T, K), sorted_token_ids=torch.empty(cap),
             expert_ids=torch.empty((cap + bm - 1) // bm), num_tokens_post_padded=torch.empty(1), block_m=bm)
    if fmt != "bf16":
        a.update(x_scales=torch.empty(T, K // 32),
                 w1_scales=torch.empty(moe.pack_scales_blocked_bytes(E, N, K // 32)),
                 w2_scales=torch.empty(moe.pack_scales_blocked_bytes(E, K, N // 64)))
    return a


@pytest.mark.parametrize("fmt", ["bf16", "mxfp8", "mxfp4"])
def test_matching_shapes_pass(fmt):
    moe._ffn_shapes(fmt, **_args(fmt))


@pytest.mark.parametrize("fmt,name,bad", [
    ("bf16", "w2", torch.empty(E, K, N)),                 # full N instead of N/2
    ("bf16", "w2", torch.empty(E - 1, K, N // 2)),        # fewer experts than w1
    ("bf16", "out", torch.empty(T - 1, K)),
    ("bf16", "topk_weights", torch.empty(T + 1, k)),
    ("bf16", "topk_weights", torch.empty(T * k)),
    ("bf16", "expert_ids", torch.empty(1)),
    ("bf16", "num_tokens_post_padded", torch.empty(0)),
    ("mxfp8", "x_scales", torch.empty(T, K // 16)),
    ("mxfp8", "w1_scales", torch.empty(100)),
    ("mxfp8", "w2_scales", torch.empty(100)),
    ("mxfp4", "w1", torch.empty(E, N, K)),                # unpacked weights on the packed path
    ("mxfp4", "w2", torch.empty(E, K, N // 2)),
    ("bf16", "w2", torch.empty(E, K, N // 2, device="meta")),   # another device
])
def test_mismatches_are_rejected(fmt, name, bad):
    a = _args(fmt)
    a[name] = bad
    with pytest.raises(ValueError):
        moe._ffn_shapes(fmt, **a)


def test_odd_n_is_rejected():
    a = _args("bf16")
    a["w1"] = torch.empty(E, N + 1, K)
    with pytest.raises(ValueError):
        moe._ffn_shapes("bf16", **a)
