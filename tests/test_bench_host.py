"""bench.py's host-side pieces on CPU: the cost model's bytes per weight value for every weight format,
and the option checks."""
import numpy as np
import pytest

import bench
import workloads as W

PEAKS = {"hbm_gbs": 6539.9, "bf16_tflops": 1617.4}


@pytest.mark.parametrize("name,b", [("C2", 2.0), ("C3", 1.0 + 1.0 / 32.0), ("C3F4", 0.5 + 1.0 / 32.0)])
def test_weight_bytes_per_value(name, b):
    sh = W.shape(name, 64)
    ids = np.tile(np.arange(sh.top_k, dtype=np.int32), (sh.T, 1))     # top_k touched experts
    cm = bench.cost_model(sh, ids, PEAKS)
    assert cm["touched"] == sh.top_k
    assert cm["bytes_w"] == pytest.approx(sh.top_k * 1.5 * sh.N * sh.K * b)
    assert cm["flops"] == pytest.approx(3.0 * sh.T * sh.top_k * sh.K * sh.N)


def test_mxfp4_roofline_halves_the_weight_time():
    sh8, sh4 = W.shape("C3", 64), W.shape("C3F4", 64)
    ids = np.tile(np.arange(8, dtype=np.int32), (64, 1))
    t8 = bench.cost_model(sh8, ids, PEAKS)["t_hbm"]
    t4 = bench.cost_model(sh4, ids, PEAKS)["t_hbm"]
    assert t4 / t8 == pytest.approx((0.5 + 1 / 32) / (1 + 1 / 32))


def test_option_checks():
    with pytest.raises(SystemExit):
        bench.parse_args(["--shared", "1"])            # shared experts come with the router
    with pytest.raises(SystemExit):
        bench.parse_args(["--router", "--shared", "-1"])
    a = bench.parse_args(["--router", "--shared", "2", "--workload", "C3F4", "--tokens", "64"])
    assert a.router and a.shared == 2 and a.workload == "C3F4"
