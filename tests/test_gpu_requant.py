"""Byte-level parity of the on-chip mxfp8 requant of the SwiGLU intermediate.

"Prime Flash MoE: Fused MoE Kernels for Blackwell", intro: the intermediate is requantised to mxfp8
on chip before the down projection; Scale layout (mxfp8): e4m3 values with one e8m0 scale per 32
(the OCP MX rule: scale 2^(floor(log2 amax) - 8), e4m3 round-to-nearest-even, saturation at 448).

After an mxfp8 call the caller-owned workspace holds what the gate/up phase wrote: ``act`` (one
row of N/2 e4m3 codes per planner row, at offset 0) and ``act_sf`` (the e8m0 scales in 512-byte
blocked tiles, one per (planner block, 128 intermediate columns), at the next 1024-byte boundary;
row r of a block and scale c of a tile at byte (r % 32) * 16 + (r / 32) * 4 + c).  Both are read
back and compared with the oracle's OCP quantiser applied to the oracle's fp32 SwiGLU values.

The GPU's fp32 SwiGLU values differ from the oracle's (double sums rounded once) by accumulation
order and the fast exp, a few parts in 1e6 of the block maximum.  So a scale byte may differ only
in a block whose amax lies within 2^-14 (relative) of a power of two, and a code only where the
exact scaled value lies within 2^-14 of the block maximum from the rounding midpoint of the two
codes, which must be neighbours on the e4m3 grid, or where both codes are zeros of opposite sign
(the exact value then lies within that distance of zero).  Every other byte must be equal; the number of
exempt bytes is printed and must stay below 1e-3 of those compared.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import coverage_sample, to_dev

pytestmark = pytest.mark.gpu

_E4M3 = np.array([oracle.e4m3_to_double(c) for c in range(256)])  # the oracle's pinned decoder
_FINITE = np.sort(np.unique(_E4M3[np.isfinite(_E4M3)]))
TAU = 2.0 ** -14


def _round_up(a, b):
    return (a + b - 1) // b * b


def _gpu_requant(sh, inp):
    """Runs moe_align + the fused mxfp8 / MXFP4 forward and returns (sorted_ids, act, act_sf) read
    back from the workspace."""
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    ids, tw = to_dev(inp["topk_ids"]), to_dev(inp["topk_weights"])
    s_ids, e_ids, ntpp = moe.moe_align(ids, sh.E, sh.block_m)
    x, xs, w1, w2 = (to_dev(inp[n]) for n in ("x", "x_scales", "w1", "w2"))
    s1 = moe.pack_scales_blocked(to_dev(inp["w1_scales"]))
    s2 = moe.pack_scales_blocked(to_dev(inp["w2_scales"]))
    dt = moe.DTYPE_MXFP4 if sh.dtype == "mxfp4" else moe.DTYPE_MXFP8
    ws = torch.empty(moe.moe_workspace_bytes(dt, sh.T, sh.K, sh.N, sh.E, sh.top_k, sh.block_m), dtype=torch.uint8,
                     device="cuda")
    ws.fill_(0xA5)  # poison: a byte the kernel should have written and did not shows up
    out = torch.empty((sh.T, sh.K), dtype=torch.bfloat16, device="cuda")
    fwd = moe.fused_moe_mxfp4 if sh.dtype == "mxfp4" else moe.fused_moe_mxfp8
    fwd(x, xs, w1, s1, w2, s2, s_ids, e_ids, ntpp, tw, out, sh.block_m, workspace=ws)
    moe.moe_device_status()
    cap_rows = _round_up(sh.R + sh.E * (sh.block_m - 1), sh.block_m)
    act_bytes = cap_rows * sh.I
    sf_off = _round_up(act_bytes, 1024)
    n_jt = (sh.I + 127) // 128
    sf_bytes = (cap_rows // sh.block_m) * n_jt * 512
    host = ws[: sf_off + sf_bytes].cpu().numpy()
    return s_ids.cpu().numpy(), host[:act_bytes].reshape(cap_rows, sh.I), host[sf_off:sf_off + sf_bytes], n_jt


def check_requant(sh, inp, toks):
    sorted_ids, act, act_sf, n_jt = _gpu_requant(sh, inp)
    af = oracle.mx_intermediate(inp["x"], inp["x_scales"], inp["w1"], inp["w1_scales"], inp["topk_ids"],
                                tokens=toks, fp4=sh.dtype == "mxfp4")           # (n, k, I) fp32
    k, I, bm = sh.top_k, sh.I, sh.block_m
    pos = np.full(sh.R, -1, dtype=np.int64)
    live = np.nonzero(sorted_ids >= 0)[0]
    pos[sorted_ids[live]] = live
    routes = (toks[:, None].astype(np.int64) * k + np.arange(k)[None, :]).reshape(-1)
    e = inp["topk_ids"].reshape(-1)[routes]
    keep = (e >= 0) & (e < sh.E)
    assert np.all(pos[routes[keep]] >= 0), "a valid route has no planner row"
    p = pos[routes[keep]]
    v = af.reshape(-1, I)[keep]                                                 # oracle fp32 rows
    codes_o, sf_o = oracle.mx_quantize(v)
    codes_g = act[p]                                                            # GPU rows
    b, rr = p // bm, p % bm
    g = np.arange(I // 32)
    sf_idx = ((b[:, None] * n_jt + g[None, :] // 4) * 512 + (rr[:, None] % 32) * 16 + (rr[:, None] // 32) * 4
              + g[None, :] % 4)
    sf_g = act_sf[sf_idx]

    # scale bytes
    amax = np.abs(v.reshape(len(v), -1, 32)).max(axis=2)
    m, _ = np.frexp(amax.astype(np.float64))
    near_pow2 = (amax > 0) & ((2 * m < 1 + TAU) | (2 * m > 2 - 2 * TAU))
    sf_diff = sf_g != sf_o
    bad_sf = sf_diff & ~(near_pow2 & (np.abs(sf_g.astype(int) - sf_o.astype(int)) == 1))
    assert not bad_sf.any(), (f"{int(bad_sf.sum())} of {sf_o.size} scale bytes differ from the OCP rule, e.g. gpu "
                              f"{sf_g[bad_sf][:8]} oracle {sf_o[bad_sf][:8]}")

    # codes, in blocks whose scale agrees
    same = np.repeat(~sf_diff, 32, axis=1)
    diff = (codes_g != codes_o) & same
    exempt = signed_zeros = 0
    if diff.any():
        r_i, c_i = np.nonzero(diff)
        scale = np.ldexp(1.0, sf_o[r_i, c_i // 32].astype(np.int64) - 127)
        exact = v[r_i, c_i].astype(np.float64) / scale
        blockmax = amax[r_i, c_i // 32].astype(np.float64) / scale
        vo, vg = _E4M3[codes_o[r_i, c_i]], _E4M3[codes_g[r_i, c_i]]
        neighbours = np.abs(np.searchsorted(_FINITE, vo) - np.searchsorted(_FINITE, vg)) == 1
        near_mid = np.abs(exact - 0.5 * (vo + vg)) <= TAU * blockmax
        # +0 and -0: a value that rounds to zero keeps the sign of an fp32 value within rounding
        # noise of zero, which the two sides may see with opposite signs
        zero_sign = (vo == 0) & (vg == 0) & (np.abs(exact) <= TAU * blockmax)
        ok = np.isfinite(vg) & ((neighbours & near_mid) | zero_sign)
        assert ok.all(), (f"{int((~ok).sum())} e4m3 codes differ away from a rounding midpoint, e.g. exact "
                          f"{exact[~ok][:4]} oracle {vo[~ok][:4]} gpu {vg[~ok][:4]}")
        exempt = int(ok.sum())
        signed_zeros = int(zero_sign.sum())
    compared = int(same.sum())
    print(f"REQUANT {sh.name} T={sh.T} routes={len(v)} scale bytes={sf_o.size} (exempt near 2^n: "
          f"{int(sf_diff.sum())}) codes={compared} (exempt: {exempt}, of which signed zeros {signed_zeros})")
    assert sf_diff.sum() <= 1e-3 * sf_o.size and exempt <= 1e-3 * max(compared, 1)


def small(dtype, T, K, N, E, top_k, block_m):
    return W.Shape(name="S", dtype=dtype, T=T, K=K, N=N, E=E, top_k=top_k, block_m=block_m)


@pytest.mark.parametrize("sh", [
    small("mxfp8", 200, 256, 512, 8, 2, 128),
    small("mxfp8", 90, 256, 768, 6, 3, 32),      # 3 intermediate tiles, 32-row blocks
    small("mxfp8", 12, 1024, 512, 4, 2, 128),    # split-K: written by the reduction kernel
    small("mxfp4", 200, 512, 256, 8, 2, 64),     # MXFP4 weights, same requant
], ids=lambda s: f"{s.dtype}-T{s.T}-K{s.K}-N{s.N}-bm{s.block_m}")
def test_requant_bytes_small(sh):
    inp = W.inputs(sh, seed=13)
    check_requant(sh, inp, np.arange(sh.T, dtype=np.int32))


def test_requant_bytes_c3_t2048():
    """C3 at T=2048 (mxfp8, K=4096, N/2=2048, E=288, top-8), a 512-token coverage sample."""
    sh = W.shape("C3", 2048)
    ids, tw = W.routing(sh)
    w1, s1 = W.mxfp8_weights(sh, "w1")
    w2, s2 = W.mxfp8_weights(sh, "w2")
    x, xs = W.mx_quantize_inputs(W.x_f32(sh))
    inp = dict(x=x, x_scales=xs, w1=w1, w1_scales=s1, w2=w2, w2_scales=s2, topk_ids=ids, topk_weights=tw)
    check_requant(sh, inp, coverage_sample(sh, ids, 512))
