"""bench.py's GEMM roofline arithmetic (host only)."""
import numpy as np

import bench
import synth

PEAKS = {"hbm_gbs": 6446.9, "bf16_tflops": 1668.7}


def test_gptoss_layer_is_tensor_bound_and_decode_is_hbm_bound():
    wl = synth.WORKLOADS["gptoss_uniform"]
    b = bench.gemm_bounds(wl, np.full(wl.E, wl.S // wl.E), False, PEAKS)
    for proj in ("gate_up", "down"):
        assert b[proj]["t_tensor"] > b[proj]["t_hbm"]
        # balanced experts above the ridge: the per-expert bound is the tensor time
        np.testing.assert_allclose(b[proj]["t_per_expert"], b[proj]["t_tensor"], rtol=1e-12)
    wl = synth.WORKLOADS["dsr1_decode"]
    counts = np.zeros(wl.E, np.int64)
    counts[: wl.S // 4] = 4  # 256 experts, 1024 rows: every fourth row block on one expert
    b = bench.gemm_bounds(wl, counts, True, PEAKS)
    assert b["gate_up"]["t_hbm"] > 10 * b["gate_up"]["t_tensor"]


def test_bytes_count_active_experts_and_the_gathered_rows_once():
    wl = synth.Workload("t", T=64, H=128, I=256, E=8, k=2, R=2, dtype="bf16", seed=0)
    counts = np.array([0, 40, 0, 30, 0, 58, 0, 0])
    assert counts.sum() == wl.S
    rows = bench.gemm_bounds(wl, counts, False, PEAKS)["gate_up"]
    gath = bench.gemm_bounds(wl, counts, True, PEAKS)["gate_up"]
    w = 3 * 2 * wl.H * wl.I * 2  # three active experts, gate + up, bf16
    assert rows["bytes"] == w + wl.S * wl.H * 2 + wl.S * wl.I * 2
    assert gath["bytes"] == w + wl.T * wl.H * 2 + wl.S * wl.I * 2
    assert rows["flops"] == 4.0 * wl.S * wl.H * wl.I
    # sum_e max(a_e, b_e) >= max(sum_e a_e, sum_e b_e): never below either global bound
    assert rows["t_per_expert"] >= max(rows["t_tensor"], rows["t_hbm"]) * (1 - 1e-12)
    down = bench.gemm_bounds(wl, counts, True, PEAKS)["down"]
    assert down["bytes"] == 3 * wl.I * wl.H * 2 + wl.S * wl.I * 2 + wl.S * wl.H * 2
