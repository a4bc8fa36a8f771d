"""The bench's cost model and launch count on the CPU: the algorithmic bytes and flops per stage
follow the per-unit definitions (x read once by the router, expert ids read once by the grouping,
each used expert's weights streamed once, the token rows gathered once, h written and read once,
y written and read once), so the roofline fractions divide the right numbers."""
import numpy as np

import bench
from expert_dispatch_gate_b200 import workloads as W


def test_stage_costs_fine_grained_per_unit_definitions():
    wl = W.WORKLOADS["fine"]
    T, H, E, k, I = 4096, 4096, 256, 8, 2048
    assert (wl.T, wl.H, wl.E, wl.k, wl.I, wl.dtype) == (T, H, E, k, I, "bf16")
    counts = np.full(E, 128, dtype=np.int64)  # every expert used, 32768 kept
    A = T * k
    c = bench.stage_costs(wl, counts, hbm_peak=6550.4, tc_peak=1390.0)
    assert c["route"]["bytes"] == T * H * 2 + H * E * 2 + T * k * 8 == 35_913_728
    assert c["route"]["flops"] == 2 * T * H * E
    assert c["align"]["bytes"] == A * 4 + A * 9 + E * 8
    weights = E * 3 * H * I * 2
    assert weights == 12_884_901_888
    assert c["gemm1"]["bytes"] == E * 2 * H * I * 2 + A * H * 2 + A * I * 2
    assert c["gemm2"]["bytes"] == E * I * H * 2 + A * I * 2 + A * H * 2
    assert c["gemm1"]["flops"] + c["gemm2"]["flops"] == 6 * A * H * I
    assert c["combine"]["bytes"] == A * H * 2 + T * k * 8 + T * H * 2
    assert abs(c["route"]["t_hbm_us"] - 35_913_728 / 6550.4e9 * 1e6) < 1e-9
    assert abs(c["gemm1"]["t_tc_us"] - 4 * A * H * I / 1390e12 * 1e6) < 1e-9


def test_stage_costs_count_only_used_experts_and_kept_rows():
    wl = W.WORKLOADS["skewed"]  # T=32768 H=2048 E=64 k=6 I=1408, Zipf logit bias
    counts = np.zeros(64, dtype=np.int64)
    counts[:10] = 3840  # ten experts at capacity, the rest unused
    c = bench.stage_costs(wl, counts, hbm_peak=6550.4, tc_peak=1390.0)
    kept = 38400
    assert c["gemm1"]["bytes"] == 10 * 2 * 2048 * 1408 * 2 + kept * 2048 * 2 + kept * 1408 * 2
    assert c["route"]["bytes"] == 32768 * 2048 * 2 + 2048 * 64 * 2 + 64 * 4 + 32768 * 6 * 8


def test_stage_costs_fp8_weights_are_one_byte_plus_channel_scales():
    wl = W.WORKLOADS["fine"]
    counts = np.full(256, 128, dtype=np.int64)
    c8 = bench.stage_costs(wl, counts, 6550.4, 1390.0, fp8_weights=True)
    c16 = bench.stage_costs(wl, counts, 6550.4, 1390.0)
    assert c16["gemm1"]["bytes"] - c8["gemm1"]["bytes"] == 256 * 2 * 4096 * 2048 - 256 * 2 * 2048 * 4
    assert c16["gemm2"]["bytes"] - c8["gemm2"]["bytes"] == 256 * 2048 * 4096 - 256 * 4096 * 4


def test_launches_per_step():
    # router gate GEMM + top-k, one grouping launch, the row copy, two expert GEMMs, the combine
    assert bench.launches_per_step(W.WORKLOADS["fine"]) == 7
    assert bench.launches_per_step(W.WORKLOADS["decode"].with_tokens(256)) == 7
    assert bench.launches_per_step(W.WORKLOADS["decode"].with_tokens(1)) == 7
    # skewed: E = 64 with the hidden dimension in one K range (T = 32768) runs the gate GEMM and
    # the top-k as one kernel; 196608 assignments group in one cooperative launch; every bf16
    # layer makes the row copy, whatever I
    assert bench.route_ksplit(32768, 2048, 64) == 1
    # I = 1408 = 5 x 256 + 128: GEMM1's last 128 features run as a second, single-CTA launch
    assert bench.launches_per_step(W.WORKLOADS["skewed"]) == 1 + 1 + 1 + 3 + 1
    # fine-grained at T = 32768: one K range on CTA pairs, gate GEMM and top-k fused
    assert bench.route_ksplit(32768, 4096, 256) == 1
    assert bench.launches_per_step(W.WORKLOADS["fine"].with_tokens(32768)) == 1 + 1 + 1 + 2 + 1
    # a short E = 64 batch splits K, so gate GEMM and top-k run separately
    assert bench.route_ksplit(4096, 2048, 64) == 4
    assert bench.launches_per_step(W.WORKLOADS["skewed"].with_tokens(4096)) == 2 + 1 + 1 + 3 + 1
    # W8A8: the token rows and the SwiGLU rows are quantised by one launch each
    assert bench.launches_per_step(W.WORKLOADS["fine"], "w8a8") == 9
    # tiny f32: one fused CUDA-core router kernel
    assert bench.launches_per_step(W.WORKLOADS["tiny"]) == 1 + 1 + 0 + 2 + 1


def test_reference_arm_line_matches_our_config_and_reports_its_own_wall_time():
    """The reference arm (the oracle on the host) prints the same config keys as the GPU arm,
    the measured wall time of its sample as ms_per_step, and the extrapolation separately."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                       cwd=bench.ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    wl = W.WORKLOADS["tiny"]
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["config"] == bench.layer_config(wl, 64, 1)
    assert line["ms_per_step"] <= line["ms_per_step_extrapolated_to_T"] * 10
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert "8 sampled tokens" in line["cpu_baseline"]["sample"]
