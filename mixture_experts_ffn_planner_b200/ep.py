"""Expert-parallel forward over the ranks of a torch.distributed group.

The multi-GPU setting of the pages ("[SM90] Ring-buffered FP8 MegaMoE with a lag-ordered L1/L2 schedule"
and DeepGEMM #411 "SM90 FP8 x MXFP4 MegaMoE": EP8 dispatch, routed experts, combine): the experts are
sharded over the G ranks of a group (rank r owns experts [r*E/G, (r+1)*E/G)); every rank sends each of
its routed rows to the rank that owns the route's expert (dispatch, all-to-all), runs the local fused
MoE forward on the rows it receives, and the weighted results travel back (combine, all-to-all) to be
summed per token in route order.

This is the collective form of that step: the exchanges are ``all_to_all_single`` of the group's
backend (NCCL over NVLink between B200s, gloo between CPU processes), and the local forward is a
callable -- on GPUs the fused kernels of this library (``local_ffn_bf16``).  Dispatch and combine are
not fused into the GEMM kernels here.

Route order: a token's routes are summed in their top-k order on the token's own rank, so the result
does not depend on the number of ranks or on their scheduling.
"""
from __future__ import annotations

from typing import Callable

__all__ = ["ep_forward", "local_ffn_bf16", "owner_of"]


def owner_of(expert_ids, E: int, world: int):
    """Rank that owns each expert id (experts split into `world` equal contiguous ranges); -1 for ids
    outside [0, E)."""
    import torch

    per = E // world
    valid = (expert_ids >= 0) & (expert_ids < E)
    return torch.where(valid, torch.div(expert_ids, per, rounding_mode="floor"), torch.full_like(expert_ids, -1))


def ep_forward(x, topk_ids, topk_weights, E: int, local_ffn: Callable, group=None, x_scales=None):
    """Expert-parallel MoE forward of this rank's tokens.

    x (T, K) rows of this rank (bf16 values, or e4m3 codes as uint8); topk_ids (T, k) int32 global
    expert ids (ids outside [0, E) route nowhere); topk_weights (T, k) fp32.  x_scales (T, K/32) uint8
    e8m0, for e4m3 rows: each row's scales travel with it.  local_ffn(rows (M, K), local_expert (M,)
    int32, weight (M,) fp32[, row_scales (M, K/32) when x_scales is given]) returns the weighted expert
    outputs (M, K) of the rows this rank received (any float dtype).
    Returns out (T, K) in local_ffn's dtype: for every token the sum, in route order, of its routes'
    weighted expert outputs.  E must be a multiple of the group size.
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if E % world:
        raise ValueError(f"E={E} experts do not split evenly over {world} ranks")
    per = E // world
    T, k = topk_ids.shape
    K = x.shape[1]
    dev = x.device

    ids = topk_ids.reshape(-1).to(torch.int64)
    dest = owner_of(ids, E, world)
    live = torch.nonzero(dest >= 0).reshape(-1)               # route indices t*k + j that go somewhere
    order = live[torch.argsort(dest[live], stable=True)]       # grouped by destination rank
    send_counts = torch.bincount(dest[live], minlength=world).to(torch.int64)

    # sizes first, then the rows and their per-route metadata
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    M = sum(rc)
    rows_out = x[torch.div(order, k, rounding_mode="floor")].contiguous()
    local_e_out = (ids[order] - dest[order] * per).to(torch.int32)
    w_out = topk_weights.reshape(-1)[order].contiguous()
    rows_in = torch.empty((M, K), dtype=x.dtype, device=dev)
    local_e_in = torch.empty(M, dtype=torch.int32, device=dev)
    w_in = torch.empty(M, dtype=w_out.dtype, device=dev)
    dist.all_to_all_single(rows_in, rows_out, rc, sc, group=group)
    dist.all_to_all_single(local_e_in, local_e_out, rc, sc, group=group)
    dist.all_to_all_single(w_in, w_out, rc, sc, group=group)
    if x_scales is not None:
        sc_out = x_scales[torch.div(order, k, rounding_mode="floor")].contiguous()
        sc_in = torch.empty((M, x_scales.shape[1]), dtype=x_scales.dtype, device=dev)
        dist.all_to_all_single(sc_in, sc_out, rc, sc, group=group)
        y_in = local_ffn(rows_in, local_e_in, w_in, sc_in)
    else:
        y_in = local_ffn(rows_in, local_e_in, w_in)           # (M, K) weighted outputs of received routes
    y_back = torch.empty((len(order), K), dtype=y_in.dtype, device=dev)
    dist.all_to_all_single(y_back, y_in.contiguous(), sc, rc, group=group)

    # combine: every route's result at its (token, slot), then the slots summed in route order
    per_route = torch.zeros((T * k, K), dtype=y_back.dtype, device=dev)
    per_route[order] = y_back
    per_route = per_route.view(T, k, K)
    out = per_route[:, 0].clone()
    for j in range(1, k):
        out += per_route[:, j]
    return out


def local_ffn_bf16(w1_local, w2_local, block_m: int = 128):
    """The local forward for ep_forward on GPUs: this rank's experts (E_local, N, K) / (E_local, K, N/2)
    bf16 through moe_align + fused_moe_bf16, one route per received row with its routing weight.
    Returns fp32 (the bf16 result of each route, which the combine sums in fp32)."""
    import torch

    from . import fused_moe_bf16, moe_align

    E_local = w1_local.shape[0]

    def run(rows, local_expert, weight):
        M, K = rows.shape
        out = torch.empty((M, K), dtype=torch.bfloat16, device=rows.device)
        if M == 0:
            return out.float()
        s_ids, e_ids, ntpp = moe_align(local_expert.reshape(M, 1).contiguous(), E_local, block_m)
        fused_moe_bf16(rows.contiguous(), w1_local, w2_local, s_ids, e_ids, ntpp,
                       weight.reshape(M, 1).float().contiguous(), out, block_m)
        return out.float()

    return run
