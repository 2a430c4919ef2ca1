"""Pins of the oracle's mxfp8 SwiGLU intermediate (``oracle.mx_intermediate``), the fp32 values
the on-chip requant starts from ("Prime Flash MoE: Fused MoE Kernels for Blackwell", intro: the
intermediate is requantised to mxfp8 on chip before the down projection).

* Dense top-1 case against torch float64: fp32( silu(w1_gate x) * (w1_up x) ) with the exactly
  dequantised operands, row for row.
* Consistency with the pinned forward: requantising the exported rows (the pinned OCP quantiser),
  projecting them with torch float64 through the dequantised w2 and summing with the routing
  weights gives the forward's unrounded output; this fixes the row order (token, then route) and
  the zero rows of routes to no expert.
"""
import numpy as np
import torch

import oracle
import workloads as W


def _deq(codes, scales):
    """e4m3 codes (..., L) and e8m0 scales (..., L/32) -> float64, through torch's float8 type."""
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)
    s = torch.pow(2.0, torch.from_numpy(scales.astype(np.float64)) - 127.0)
    return (v.reshape(*v.shape[:-1], -1, 32) * s[..., None]).reshape(v.shape)


def _case(T=9, K=128, N=192, E=3, top_k=2, seed=5):
    sh = W.Shape(name="S", dtype="mxfp8", T=T, K=K, N=N, E=E, top_k=top_k, block_m=32)
    inp = W.inputs(sh, seed=seed)
    return sh, inp


def test_dense_top1_against_torch():
    sh, inp = _case(top_k=1, E=1)
    act = oracle.mx_intermediate(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["topk_ids"])
    x = _deq(inp["x"], inp["x_scales"])
    w1 = _deq(inp["w1"][0], inp["w1_scales"][0])
    h = torch.nn.functional.linear(x, w1)
    ref = (torch.nn.functional.silu(h[:, : sh.I]) * h[:, sh.I:]).to(torch.float32).numpy()
    np.testing.assert_allclose(act[:, 0, :], ref, rtol=2e-7, atol=1e-30)


def test_rows_reproduce_the_forward():
    sh, inp = _case()
    ids = inp["topk_ids"].copy()
    ids[2, 1] = -1          # a route to no expert
    ids[4, 0] = sh.E        # an id past the last expert
    toks = np.array([0, 2, 3, 4, 8], dtype=np.int32)
    poison = np.full((len(toks), sh.top_k, sh.I), np.nan, dtype=np.float32)
    act = oracle.mx_intermediate(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], ids, tokens=toks,
                                 out=poison)
    assert np.all(act[1, 1] == 0) and np.all(act[3, 0] == 0)
    codes, scales = oracle.mx_quantize(act)
    a = _deq(codes, scales)
    _, ref = oracle.fused_moe_mxfp8(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["w2"],
                                    inp["w2_scales"], ids, inp["topk_weights"], tokens=toks, unrounded=True)
    w2 = _deq(inp["w2"], inp["w2_scales"])
    for n, t in enumerate(toks):
        acc = torch.zeros(sh.K, dtype=torch.float64)
        for j in range(sh.top_k):
            e = int(ids[t, j])
            if 0 <= e < sh.E:
                acc += float(inp["topk_weights"][t, j]) * (w2[e] @ a[n, j])
        np.testing.assert_allclose(ref[t], acc.numpy(), rtol=1e-12, atol=1e-12)
