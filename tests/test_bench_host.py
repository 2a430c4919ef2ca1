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


def test_cpu_threads_option():
    with pytest.raises(SystemExit):
        bench.parse_args(["--cpu-threads", "-1"])
    assert bench.oracle_threads(bench.parse_args(["--cpu-threads", "1"]).cpu_threads) == 1
    assert bench.oracle_threads(0) >= 1


def _m(warm):
    return {"ms_step": 2.0, "warm_ms_step": warm, "plan_ms": 0.01, "p1_ms": 1.2, "p2_ms": 0.7, "cb_ms": 0.05,
            "clocks": None, "launches": 20}


def test_warm_time_is_reported_beside_the_cold_one():
    sh = W.shape("C1", 64)
    ids = np.tile(np.arange(sh.top_k, dtype=np.int32), (sh.T, 1))
    cm = bench.cost_model(sh, ids, PEAKS)
    cold = bench.result_line(sh, cm, _m(1.5), 1, 4, 3, PEAKS, "measured", True)
    assert cold["us_per_call"] == pytest.approx(2000.0)            # the reported value stays the cold one
    assert cold["warm"]["us_per_call"] == pytest.approx(1500.0)
    assert "not flushed" in cold["warm"]["l2"]
    assert "warm" not in bench.result_line(sh, cm, _m(None), 1, 4, 3, PEAKS, "measured", False)


def test_full_algorithmic_bytes():
    sh = W.shape("C2", 64)                                 # bf16, block_m 128
    ids = np.tile(np.arange(sh.top_k, dtype=np.int32), (sh.T, 1))
    cm = bench.cost_model(sh, ids, PEAKS)
    R = sh.T * sh.top_k
    cap = R + sh.E * (sh.block_m - 1)
    want = (cm["bytes_w"] + 2 * sh.T * sh.K + 2 * sh.T * sh.K + 8 * R + 4 * cap
            + 4 * ((cap + sh.block_m - 1) // sh.block_m) + 4)
    assert cm["bytes_full"] == pytest.approx(want)
    assert cm["bytes_full"] > cm["bytes_w"]


def test_roofline_follows_the_dominant_kernel():
    sh = W.shape("C5", 64)
    ids = np.tile(np.arange(sh.top_k, dtype=np.int32), (sh.T, 1))
    peaks = dict(PEAKS, mxfp8_tflops=2928.7)
    cm = bench.cost_model(sh, ids, peaks)
    m = {"p1_ms": 0.01, "p2_ms": 0.05, "cb_ms": 0.002, "plan_ms": 0.003}
    r = bench.roofline_of(sh, cm, m, peaks, "measured")
    assert r["phase"] == "down" and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(cm["kernels"]["down"]["bytes"] / 0.05e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"])
    m = {"p1_ms": 0.08, "p2_ms": 0.05, "cb_ms": 0.002, "plan_ms": 0.003}
    assert bench.roofline_of(sh, cm, m, peaks, "measured")["phase"] == "gate_up"


def test_mxfp8_peak_comes_from_the_committed_measurement():
    peaks, _ = bench.load_peaks()
    assert peaks["mxfp8_tflops"] > peaks["bf16_tflops"]
    assert "profiles/tensor_peak_mxfp8.md" in peaks["mxfp8_source"]
    assert bench.tensor_peak(W.shape("C3", 64), peaks) == peaks["mxfp8_tflops"]
    assert bench.tensor_peak(W.shape("C3F4", 64), peaks) == peaks["mxfp8_tflops"]
    assert bench.tensor_peak(W.shape("C2", 64), peaks) == peaks["bf16_tflops"]


def test_sweep_and_headline_options():
    a = bench.parse_args([])
    assert a.workload == "C4" and a.tokens == 8192 and not a.sweep
    assert bench.parse_args(["--sweep", "--sweep-workloads", "C1,C5"]).sweep
    with pytest.raises(SystemExit):
        bench.parse_args(["--sweep", "--gpus", "2"])
    with pytest.raises(SystemExit):
        bench.parse_args(["--sweep", "--sweep-workloads", "C9"])
    assert bench.parse_args(["--no-graph"]).no_graph


def test_kernel_traffic_is_dropped_when_its_source_changes(tmp_path, monkeypatch):
    """A profile's DRAM bytes count only while the source file it names is unchanged."""
    import hashlib

    csrc = tmp_path / "mixture_experts_ffn_planner_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "small_batch.cu").write_text("kernel a")
    (csrc / "fused_moe.cu").write_text("kernel b")
    (tmp_path / "profiles").mkdir()
    sha_a = hashlib.sha256(b"kernel a").hexdigest()
    sha_b = hashlib.sha256(b"kernel b").hexdigest()
    (tmp_path / "profiles" / "k_W.md").write_text(
        f"dram_bytes_per_launch: 1.5e9\nsource_file: small_batch.cu\nsource_sha256: {sha_a}\n")
    (tmp_path / "profiles" / "j_W.md").write_text(f"dram_bytes_per_launch: 2.5e9\nsource_sha256: {sha_b}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k", "W") == 1.5e9
    assert bench.kernel_traffic("j", "W") == 2.5e9          # no source_file: fused_moe.cu
    (csrc / "small_batch.cu").write_text("kernel a, changed")
    assert bench.kernel_traffic("k", "W") is None
    assert bench.kernel_traffic("missing", "W") is None


def test_small_batch_form_follows_the_library_switch():
    """The bench's launch count and kernel names follow fused_moe_bf16's choice of form: bf16 with K and
    N/2 multiples of 256, by default when T * top_k <= 128; forced on or off by moe_tuning.small_batch."""
    c1, c5_8, c5_64, c3 = W.shape("C1", 64), W.shape("C5", 8), W.shape("C5", 64), W.shape("C3", 64)
    assert bench.small_batch_form(c1) and bench.small_batch_form(c5_8)
    assert not bench.small_batch_form(c5_64)                 # 512 routed rows
    assert bench.small_batch_form(c5_64, 1) and not bench.small_batch_form(c1, -1)
    assert not bench.small_batch_form(c3, 1)                 # mxfp8 has no small-batch form
    odd = W.Shape(name="S", dtype="bf16", T=4, K=384, N=512, E=4, top_k=2, block_m=64)
    assert not bench.small_batch_form(odd, 1)                # K not a multiple of 256
    ids = np.zeros((c1.T, c1.top_k), np.int32)
    names = bench.cost_model(c1, ids, PEAKS)["kernels"]
    assert names["gate_up"]["ncu"] == "moe_sb_up_kernel" and names["down"]["ncu"] == "moe_sb_down_kernel"
    assert bench.cost_model(c1, ids, PEAKS, small_batch=-1)["kernels"]["gate_up"]["ncu"] == "moe_p1_kernel"
