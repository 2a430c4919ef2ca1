"""Plain torch versions of the expert-parallel device work (dispatch plan, pack, combine): the
reference the kernels are checked against on the GPU, and the ops the CPU (gloo) tests of ep_forward
run with, since CPU tensors cannot reach the kernels.  Same contract as
mixture_experts_ffn_planner_b200.ep.DeviceOps; the combine sums in y's own dtype, in route order."""
import torch

from mixture_experts_ffn_planner_b200.ep import owner_of


class TorchOps:
    def plan(self, topk_ids, E: int, world: int):
        ids = topk_ids.reshape(-1).to(torch.int64)
        dest = owner_of(ids, E, world)
        live = torch.nonzero(dest >= 0).reshape(-1)
        order = live[torch.argsort(dest[live], stable=True)]
        full = torch.full((ids.numel(),), -1, dtype=torch.int32, device=ids.device)
        full[: order.numel()] = order.to(torch.int32)
        return full, torch.bincount(dest[live], minlength=world).to(torch.int32)

    def pack(self, x, x_scales, topk_ids, topk_weights, order, n: int, E: int, world: int):
        k = topk_ids.shape[1]
        o = order[:n].to(torch.int64)
        t = torch.div(o, k, rounding_mode="floor")
        e = topk_ids.reshape(-1).to(torch.int64)[o]
        per = E // world
        return (x[t].contiguous(), None if x_scales is None else x_scales[t].contiguous(),
                (e - torch.div(e, per, rounding_mode="floor") * per).to(torch.int32),
                topk_weights.reshape(-1)[o].contiguous())

    def combine(self, y, order, n: int, T: int, top_k: int):
        per_route = torch.zeros((T * top_k, y.shape[1]), dtype=y.dtype, device=y.device)
        per_route[order[:n].to(torch.int64)] = y[:n]
        per_route = per_route.view(T, top_k, y.shape[1])
        out = per_route[:, 0].clone()
        for j in range(1, top_k):
            out += per_route[:, j]
        return out
