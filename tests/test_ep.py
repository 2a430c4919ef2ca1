"""Expert-parallel forward (ep_forward) on two and four gloo ranks on CPU.

Each rank holds its own batch; the experts are split over the ranks.  The local compute is the
oracle (tests may run it) on the rows a rank receives, so what is checked is the dispatch and the
combine: every rank's result must equal the single-process oracle on that rank's tokens with all
experts, in float64 to the last bit (routes are summed in the same order).  Covers routes that cross
ranks, routes to nowhere (id -1), a rank with no tokens, and all routes landing on one rank; on the
mxfp8 path each row's e8m0 scales travel with its e4m3 codes.
The device work on either side of the exchanges (plan, pack, combine) runs as the plain torch ops of
tests/ep_reference_ops.py here, since CPU tensors cannot reach the kernels; the kernels are checked
against those same ops on the GPU (tests/test_gpu_ep.py).  The GPU ranks of this path (NCCL between
B200s) are not exercised here: every GPU run here has one GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

K, N, E = 64, 128, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weights():
    import workloads as W

    rng = np.random.default_rng(42)
    w1 = W.f32_to_bf16_bits((rng.standard_normal((E, N, K)) / np.sqrt(K)).astype(np.float32))
    w2 = W.f32_to_bf16_bits((rng.standard_normal((E, K, N // 2)) / np.sqrt(N // 2)).astype(np.float32))
    return w1, w2


def _batch(rank, T, k, mode):
    import workloads as W

    rng = np.random.default_rng(100 + rank)
    x = W.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    if mode == "one_rank":
        ids = np.tile(np.array([[2, 3]], np.int32), (T, 1))      # experts of rank 1 only
    elif T == 0:
        ids = np.zeros((0, k), np.int32)
    else:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        ids[0, -1] = -1                                           # a route to nowhere
    w = rng.random((T, k)).astype(np.float32) + 0.1
    return x, ids, w


def _mx(a):
    import workloads as W

    return W.mx_quantize_inputs(W.bf16_bits_to_f32(a))


def _worker(rank, world, port, mode, results, fmt="bf16"):
    import datetime

    import torch.distributed as dist

    import oracle
    import workloads as W
    from mixture_experts_ffn_planner_b200.ep import ep_forward
    from tests.ep_reference_ops import TorchOps

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w1, w2 = _weights()
        per = E // world
        lo = rank * per
        T = 0 if (mode == "empty_rank" and rank == 0) else 9 + 4 * rank
        x, ids, tw = _batch(rank, T, 2, mode)
        if fmt == "mxfp8":
            (w1q, w1s), (w2q, w2s) = _mx(w1), _mx(w2)
            xq, xs = _mx(x) if T else (np.zeros((0, K), np.uint8), np.zeros((0, K // 32), np.uint8))

        def local_ffn(rows, local_e, weight, row_scales=None):
            M = rows.shape[0]
            if M == 0:
                return torch.zeros((0, K), dtype=torch.float64)
            le = local_e.numpy().reshape(M, 1).astype(np.int32)
            wt = weight.numpy().reshape(M, 1).astype(np.float32)
            if fmt == "mxfp8":
                y = oracle.fused_moe_mxfp8(rows.numpy(), row_scales.numpy(), w1q[lo:lo + per], w1s[lo:lo + per],
                                           w2q[lo:lo + per], w2s[lo:lo + per], le, wt, unrounded=True)[1]
            else:
                bits = W.f32_to_bf16_bits(rows.numpy().astype(np.float32))   # exact: rows hold bf16 values
                y = oracle.fused_moe_bf16(bits, w1[lo:lo + per], w2[lo:lo + per], le, wt, unrounded=True)[1]
            return torch.from_numpy(y)

        ids_t, tw_t = torch.from_numpy(ids).reshape(T, 2), torch.from_numpy(tw).reshape(T, 2)
        if fmt == "mxfp8":
            out = ep_forward(torch.from_numpy(xq), ids_t, tw_t, E, local_ffn, x_scales=torch.from_numpy(xs),
                             ops=TorchOps())
        else:
            xt = torch.from_numpy(W.bf16_bits_to_f32(x)) if T else torch.zeros((0, K), dtype=torch.float32)
            out = ep_forward(xt, ids_t, tw_t, E, local_ffn, ops=TorchOps())
        if T:
            if fmt == "mxfp8":
                ref = oracle.fused_moe_mxfp8(xq, xs, w1q, w1s, w2q, w2s, ids, tw, unrounded=True)[1]
            else:
                ref = oracle.fused_moe_bf16(x, w1, w2, ids, tw, unrounded=True)[1]
            results[rank] = float(np.max(np.abs(out.numpy() - ref)))
        else:
            results[rank] = 0.0 if out.shape == (0, K) else -1.0
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,world,fmt", [("mixed", 2, "bf16"), ("empty_rank", 2, "bf16"), ("one_rank", 2, "bf16"),
                                             ("mixed", 4, "bf16"), ("mixed", 2, "mxfp8"), ("empty_rank", 2, "mxfp8")])
def test_ep_forward_matches_the_single_process_oracle(mode, world, fmt):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, mode, results, fmt)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(results)
    assert res == {r: 0.0 for r in range(world)}, res


def test_owner_of():
    from mixture_experts_ffn_planner_b200.ep import owner_of

    ids = torch.tensor([0, 1, 2, 3, 7, 8, -1, 4])
    assert owner_of(ids, 8, 4).tolist() == [0, 0, 1, 1, 3, -1, -1, 2]
