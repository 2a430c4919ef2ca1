"""Expert-parallel forward over the ranks of a torch.distributed group.

The multi-GPU setting of the pages ("[SM90] Ring-buffered FP8 MegaMoE with a lag-ordered L1/L2 schedule"
and DeepGEMM #411 "SM90 FP8 x MXFP4 MegaMoE": EP8 dispatch, routed experts, combine): the experts are
sharded over the G ranks of a group (rank r owns experts [r*E/G, (r+1)*E/G)); every rank sends each of
its routed rows to the rank that owns the route's expert (dispatch, all-to-all), runs the local fused
MoE forward on the rows it receives, and the weighted results travel back (combine, all-to-all) to be
summed per token in route order.

This is the collective form of that step.  The exchanges are ``all_to_all_single`` of the group's
backend (NCCL over NVLink between B200s); the device work on either side is this library's kernels
(``DeviceOps``: ``moe_ep_dispatch_plan``, ``moe_ep_dispatch_pack``, ``moe_ep_combine``), and the local
forward is a callable -- on GPUs the fused kernels (``local_ffn_bf16``, ``local_ffn_mxfp8``).
Dispatch and combine are not fused into the GEMM kernels here.

Route order: a token's routes are summed in their top-k order on the token's own rank, so the result
does not depend on the number of ranks or on their scheduling.
"""
from __future__ import annotations

from typing import Callable

__all__ = ["ep_forward", "DeviceOps", "local_ffn_bf16", "local_ffn_mxfp8", "owner_of"]


def owner_of(expert_ids, E: int, world: int):
    """Rank that owns each expert id (experts split into `world` equal contiguous ranges); -1 for ids
    outside [0, E)."""
    import torch

    per = E // world
    valid = (expert_ids >= 0) & (expert_ids < E)
    return torch.where(valid, torch.div(expert_ids, per, rounding_mode="floor"), torch.full_like(expert_ids, -1))


class DeviceOps:
    """The device work of ep_forward as this library's kernels (CUDA tensors).

    plan(topk_ids, E, world) -> (order, send_counts): the routes reaching an expert grouped by owner
        rank (stable), then -1; the group sizes.
    pack(x, x_scales, topk_ids, topk_weights, order, n, E, world) -> (rows, scales or None,
        owner-local expert ids, weights) of the first n routes of `order`.
    combine(y, order, n, T, top_k) -> out (T, K) bf16: per token the sum in route order of its routes'
        returned rows (y (n, K) bf16, row i for route order[i]); fp32 sums, one rounding."""

    def plan(self, topk_ids, E: int, world: int):
        from . import moe_ep_dispatch_plan

        return moe_ep_dispatch_plan(topk_ids, E, world)

    def pack(self, x, x_scales, topk_ids, topk_weights, order, n: int, E: int, world: int):
        from . import moe_ep_dispatch_pack

        return moe_ep_dispatch_pack(x, topk_ids, topk_weights, order, n, E, world, x_scales=x_scales)

    def combine(self, y, order, n: int, T: int, top_k: int):
        from . import moe_ep_combine

        return moe_ep_combine(y, order, n, T, top_k)


def ep_forward(x, topk_ids, topk_weights, E: int, local_ffn: Callable, group=None, x_scales=None, ops=None):
    """Expert-parallel MoE forward of this rank's tokens.

    x (T, K) rows of this rank (bf16 values, or e4m3 codes as uint8); topk_ids (T, k) int32 global
    expert ids (ids outside [0, E) route nowhere); topk_weights (T, k) fp32.  x_scales (T, K/32) uint8
    e8m0, for e4m3 rows: each row's scales travel with it.  local_ffn(rows (M, K), local_expert (M,)
    int32, weight (M,) fp32[, row_scales (M, K/32) when x_scales is given]) returns the weighted expert
    outputs (M, K) of the rows this rank received.  ops: the device work (default ``DeviceOps``, the
    library's kernels).
    Returns out (T, K): for every token the sum, in route order, of its routes' weighted expert
    outputs (bf16 with the default ops).  E must be a multiple of the group size.
    """
    import torch
    import torch.distributed as dist

    ops = DeviceOps() if ops is None else ops
    world = dist.get_world_size(group)
    if E % world:
        raise ValueError(f"E={E} experts do not split evenly over {world} ranks")
    T, k = topk_ids.shape
    K = x.shape[1]
    dev = x.device

    order, send_counts = ops.plan(topk_ids, E, world)
    # sizes first (the split sizes of the exchanges are host values), then the rows and their metadata
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    n, M = sum(sc), sum(rc)
    rows_out, sc_out, local_e_out, w_out = ops.pack(x, x_scales, topk_ids, topk_weights, order, n, E, world)
    rows_in = torch.empty((M, K), dtype=x.dtype, device=dev)
    local_e_in = torch.empty(M, dtype=torch.int32, device=dev)
    w_in = torch.empty(M, dtype=w_out.dtype, device=dev)
    dist.all_to_all_single(rows_in, rows_out, rc, sc, group=group)
    dist.all_to_all_single(local_e_in, local_e_out, rc, sc, group=group)
    dist.all_to_all_single(w_in, w_out, rc, sc, group=group)
    if x_scales is not None:
        sc_in = torch.empty((M, x_scales.shape[1]), dtype=x_scales.dtype, device=dev)
        dist.all_to_all_single(sc_in, sc_out, rc, sc, group=group)
        y_in = local_ffn(rows_in, local_e_in, w_in, sc_in)
    else:
        y_in = local_ffn(rows_in, local_e_in, w_in)           # (M, K) weighted outputs of received routes
    y_back = torch.empty((n, K), dtype=y_in.dtype, device=dev)
    dist.all_to_all_single(y_back, y_in.contiguous(), sc, rc, group=group)
    return ops.combine(y_back, order, n, T, k)


def local_ffn_bf16(w1_local, w2_local, block_m: int = 128):
    """The local forward for ep_forward on GPUs: this rank's experts (E_local, N, K) / (E_local, K, N/2)
    bf16 through moe_align + fused_moe_bf16, one route per received row with its routing weight.
    Returns each row's weighted output in bf16 (the kernels' output type)."""
    import torch

    from . import fused_moe_bf16, moe_align

    E_local = w1_local.shape[0]

    def run(rows, local_expert, weight):
        M, K = rows.shape
        out = torch.empty((M, K), dtype=torch.bfloat16, device=rows.device)
        if M == 0:
            return out
        s_ids, e_ids, ntpp = moe_align(local_expert.reshape(M, 1).contiguous(), E_local, block_m)
        fused_moe_bf16(rows.contiguous(), w1_local, w2_local, s_ids, e_ids, ntpp,
                       weight.reshape(M, 1).float().contiguous(), out, block_m)
        return out

    return run


def local_ffn_mxfp8(w1_local, w1_scales_blocked, w2_local, w2_scales_blocked, block_m: int = 128):
    """The local forward for ep_forward on GPUs with mxfp8 rows: this rank's experts as e4m3 codes
    (E_local, N, K) / (E_local, K, N/2) with their scales packed by pack_scales_blocked, through
    moe_align + fused_moe_mxfp8, one route per received row (its e4m3 codes and e8m0 scales) with its
    routing weight.  Returns each row's weighted output in bf16."""
    import torch

    from . import fused_moe_mxfp8, moe_align

    E_local = w1_local.shape[0]

    def run(rows, local_expert, weight, row_scales):
        M, K = rows.shape
        out = torch.empty((M, K), dtype=torch.bfloat16, device=rows.device)
        if M == 0:
            return out
        s_ids, e_ids, ntpp = moe_align(local_expert.reshape(M, 1).contiguous(), E_local, block_m)
        fused_moe_mxfp8(rows.contiguous(), row_scales.contiguous(), w1_local, w1_scales_blocked, w2_local,
                        w2_scales_blocked, s_ids, e_ids, ntpp, weight.reshape(M, 1).float().contiguous(), out,
                        block_m)
        return out

    return run
