"""The binding runs every C call with the device of the call's tensors current (CPU).

The library launches on the current CUDA device and builds its TMA descriptors from the tensors'
addresses, so a call whose tensors sit on another device than the current one would have the wrong
GPU read them.  These tests stand in for the GPU with duck-typed tensors on "cuda:1", a recording
``torch.cuda.device`` and a fake library that records which device was current when it was called.
"""
import contextlib
import math

import pytest
import torch

import mixture_experts_ffn_planner_b200 as moe

T, K, N, E, k, bm = 40, 256, 512, 4, 2, 64


class FakeT:
    """Just enough of a tensor for the binding's checks: shape, dtype, device, a pointer."""

    def __init__(self, shape, dtype, dev):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(dev)
        self.is_cuda = self.device.type == "cuda"

    def dim(self):
        return len(self.shape)

    def numel(self):
        return math.prod(self.shape)

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return 1 << 20


class FakeStream:
    def __init__(self, dev, handle):
        self.device = torch.device(dev)
        self.cuda_stream = handle


class FakeLib:
    def __init__(self, state):
        self.state = state

    def __getattr__(self, name):
        if name == "moe_workspace_bytes":
            return lambda *a: 4096
        if name == "moe_align_capacity":
            return lambda T_, k_, E_, bm_: T_ * k_ + E_ * (bm_ - 1)
        if name == "moe_last_error":
            return lambda: b""

        def call(*args):
            self.state["calls"].append((name, self.state["current"], args[-1]))
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    state = {"current": torch.device("cuda", 0), "calls": []}

    @contextlib.contextmanager
    def device(dev):
        prev = state["current"]
        state["current"] = torch.device(dev)
        try:
            yield
        finally:
            state["current"] = prev

    monkeypatch.setattr(torch.cuda, "device", device)
    monkeypatch.setattr(torch.cuda, "current_stream",
                        lambda dev=None: FakeStream(dev or state["current"], 100 + torch.device(dev).index))
    monkeypatch.setattr(moe, "load", lambda build_if_stale=True: FakeLib(state))
    return state


def _bf16_args(dev):
    cap = T * k + E * (bm - 1)
    return dict(x=FakeT((T, K), torch.bfloat16, dev), w1=FakeT((E, N, K), torch.bfloat16, dev),
                w2=FakeT((E, K, N // 2), torch.bfloat16, dev),
                sorted_token_ids=FakeT((cap,), torch.int32, dev),
                expert_ids=FakeT(((cap + bm - 1) // bm,), torch.int32, dev),
                num_tokens_post_padded=FakeT((1,), torch.int32, dev),
                topk_weights=FakeT((T, k), torch.float32, dev), out=FakeT((T, K), torch.bfloat16, dev),
                block_m=bm, workspace=FakeT((4096,), torch.uint8, dev))


def test_call_runs_on_the_tensors_device(fake):
    """Tensors on cuda:1 while cuda:0 is current: the C call sees cuda:1 current and gets cuda:1's stream."""
    moe.fused_moe_bf16(**_bf16_args("cuda:1"))
    assert fake["calls"] == [("fused_moe_bf16", torch.device("cuda", 1), 101)]
    assert fake["current"] == torch.device("cuda", 0)  # restored afterwards


def test_planner_and_noalloc_run_on_the_tensors_device(fake):
    ids = FakeT((T, k), torch.int32, "cuda:1")
    moe.moe_align(ids, E, bm, *[_bf16_args("cuda:1")[n] for n in ("sorted_token_ids", "expert_ids",
                                                                   "num_tokens_post_padded")])
    a = _bf16_args("cuda:1")
    a.pop("workspace")
    moe.fused_moe_bf16_noalloc(**a)
    assert [c[:2] for c in fake["calls"]] == [("moe_align", torch.device("cuda", 1)),
                                               ("fused_moe_bf16_noalloc", torch.device("cuda", 1))]


def test_stream_of_another_device_is_rejected(fake):
    with pytest.raises(ValueError, match="stream belongs to"):
        moe.fused_moe_bf16(**_bf16_args("cuda:1"), stream=FakeStream("cuda:0", 7))
    assert fake["calls"] == []


def test_explicit_stream_of_the_same_device_is_used(fake):
    moe.fused_moe_bf16(**_bf16_args("cuda:1"), stream=FakeStream("cuda:1", 77))
    assert fake["calls"] == [("fused_moe_bf16", torch.device("cuda", 1), 77)]


def test_mixed_devices_are_rejected(fake):
    a = _bf16_args("cuda:1")
    a["workspace"] = FakeT((4096,), torch.uint8, "cuda:0")
    with pytest.raises(ValueError, match="all tensors must be on"):
        moe.fused_moe_bf16(**a)
    a = _bf16_args("cuda:1")
    a["out"] = FakeT((T, K), torch.bfloat16, "cuda:0")
    with pytest.raises(ValueError, match="all tensors must be on"):
        moe.fused_moe_bf16(**a)
    assert fake["calls"] == []
