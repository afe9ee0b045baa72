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
    a = bench.host_inputs(64, 96, 128, seed_tokens=3, seed_weight=0)
    b = bench.host_inputs(64, 96, 128, seed_tokens=3, seed_weight=0)
    c = bench.host_inputs(64, 96, 128, seed_tokens=4, seed_weight=0)
    assert a["x"].shape == (64, 96) and a["w"].shape == (128, 96) and a["dy"].shape == (64, 128)
    assert a["x"].dtype == np.uint16 and a["gamma"].shape == (96,) and a["beta"].shape == (96,)
    for k in a:
        assert np.array_equal(a[k], b[k])                       # same seeds, same inputs
    assert not np.array_equal(a["x"], c["x"]) and np.array_equal(a["w"], c["w"])  # per-rank tokens, shared W
