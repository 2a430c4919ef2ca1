"""pack_scales_blocked on the GPU against the oracle's packer: bit-exact."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


def _gpu_pack(s: np.ndarray) -> np.ndarray:
    import torch
    import mixture_experts_ffn_planner_b200 as moe

    E, MN, KS = s.shape
    out = torch.full((moe.pack_scales_blocked_bytes(E, MN, KS),), 0xA5, dtype=torch.uint8, device="cuda")
    moe.pack_scales_blocked(to_dev(s), out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("E,MN,KS", [(1, 128, 4), (3, 129, 5), (2, 1, 1), (5, 300, 33), (4, 256, 128),
                                     (2, 4096, 128), (1, 7168, 96)])
def test_random(E, MN, KS):
    s = np.random.default_rng(E * 1000 + MN + KS).integers(0, 256, size=(E, MN, KS), dtype=np.uint8)
    got = _gpu_pack(s)
    np.testing.assert_array_equal(got, oracle.pack_scales_blocked(s))
    np.testing.assert_array_equal(oracle.unpack_scales_blocked(got, E, MN, KS), s)


def test_workload_weight_scales():
    """The packed w1/w2 scales of a reduced mxfp8 workload (8 experts)."""
    sh = W.shape("C3", 64, E=8)
    _, s1 = W.mxfp8_weights(sh, "w1")
    _, s2 = W.mxfp8_weights(sh, "w2")
    np.testing.assert_array_equal(_gpu_pack(s1), oracle.pack_scales_blocked(s1))
    np.testing.assert_array_equal(_gpu_pack(s2), oracle.pack_scales_blocked(s2))
