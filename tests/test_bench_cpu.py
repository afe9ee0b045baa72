"""CPU checks of bench.py's accounting: the algorithmic bytes per element that the memory-bound
rooflines divide by, the ALU-issue peak the GEMM roofline uses, and the synthetic step inputs."""
import numpy as np

import bench


def test_algorithmic_bytes_per_element():
    r, c = 65536, 4096
    n = r * c
    # quantize (bf16 in): 2 B read + 1 B code + 4 B per 1024-element block
    assert bench.bytes_quant(r, c, 2) / n == 2 + 1 + 4 / 1024
    # an INT8-in, INT8-out operator: codes and scales read once and written once
    assert bench.bytes_i8_op(r, c) / n == 2 * (1 + 4 / 1024)
    assert bench.bytes_i8_op(r, c, extra=8 * c) == bench.bytes_i8_op(r, c) + 8 * c


def test_alu_issue_peak():
    # 4 schedulers x 32 lanes per SM per clock, 148 SMs, the 1965 MHz maximum clock: 37.2 T lane-instr/s
    peak = bench.ALU_LANES_PER_CLK_PER_SM * bench.B200_SMS * bench.FALLBACK_PEAKS["sm_max_mhz"] * 1e6
    assert abs(peak / 1e12 - 37.22) < 0.01
    # two lane-instructions per output element per 32-deep block equal 2*M*N*K / 32 int8 ops
    M, N, K = 4096, 4096, 1024
    assert 2 * M * N * (K // 32) * 32 == 2 * M * N * K


def test_step_inputs_are_seeded_and_shaped():
    dims = (64, 96, 128)
    a = bench.host_inputs(3, 0, dims)
    b = bench.host_inputs(3, 0, dims)
    c = bench.host_inputs(4, 0, dims)
    assert a["x"].shape == (64, 96) and a["dy"].shape == (64, 96)
    assert a["w1"].shape == (128, 96) and a["w2"].shape == (96, 128)
    assert a["x"].dtype == np.uint16 and a["gamma"].shape == (96,) and a["beta"].shape == (96,)
    for k in a:
        assert np.array_equal(a[k], b[k])                       # same seeds, same inputs
    # per-rank tokens, shared weights
    assert not np.array_equal(a["x"], c["x"]) and np.array_equal(a["w1"], c["w1"]) and np.array_equal(a["w2"], c["w2"])


def test_step_covers_the_path_and_counts_six_gemms():
    """One step runs every operator of the path (quantize, dequantize, LayerNorm_i8, GELU_i8, the
    three GEMM modes of both linears, and the two INT8 backward operators), and its GEMM work is six
    products of 2 * M * H * F int8 ops."""
    ops = bench.GpuStep.OPS
    for name in ("quantize_x", "dequantize_dx", "layernorm_i8", "gelu_i8", "fc1_fwd", "fc2_dgrad", "fc1_wgrad",
                 "gelu_i8_bwd", "layernorm_i8_bwd"):
        assert name in ops
    assert sorted(bench.GpuStep.GEMMS) == sorted(o for o in ops if o.startswith("fc"))
    M, H, F = bench.layer_dims()
    assert (M, H, F) == (8192, 4096, 16384)
    assert 6 * 2 * M * H * F == 6597069766656


def test_traffic_record_is_reported_only_for_the_sources_it_was_taken_of(tmp_path, monkeypatch):
    """bench.py reports the dominant GEMM's DRAM traffic from profiles/gemm_traffic.json only while the
    record's content hash equals that of the current GEMM kernel sources; otherwise null."""
    import json
    import os
    from int8_fully_quantized_b200 import build_lib
    os.makedirs(tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"fc1_fwd": 211_000_000, "kernel_source_hash": build_lib.kernel_source_hash()}
    with open(tmp_path / "profiles" / "gemm_traffic.json", "w") as f:
        json.dump(rec, f)
    assert bench._load_traffic("fc1_fwd") == 211_000_000
    assert bench._load_traffic("fc2_fwd") is None          # no figure for that launch
    rec["kernel_source_hash"] = "0" * 64                      # taken of other sources
    with open(tmp_path / "profiles" / "gemm_traffic.json", "w") as f:
        json.dump(rec, f)
    assert bench._load_traffic("fc1_fwd") is None
