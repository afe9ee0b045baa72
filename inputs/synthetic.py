"""Seeded synthetic inputs shared by the CPU oracle tests, the GPU parity tests and the benchmark.

This module holds no arithmetic of the quantization method itself: it only draws random tensors
with the shapes and value distributions of the workloads (Gaussian activations with a few
outlier channels, small Gaussian weights and gradients), converts dtypes, and builds adversarial
blocks. Everything is numpy PCG64 (``np.random.default_rng(seed)``) on the host, so the identical
host buffer feeds both the oracle and the device.

The workloads stand in for the GPT2-medium and hidden-4096 transformer layers of the Jetfire
summary (atlas.scime.ai page, "Key results" and the "Measured effects" table); no dataset is used.
"Channel" means a column of an activation matrix (tokens x channels), which is where the
channel-wise outliers of the Jetfire summary ("Approach") live.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "activation", "weight", "grad", "to_bf16_bits", "bf16_bits_to_f32", "to_f16",
    "WORKLOADS", "workload", "tie_block", "adversarial_blocks",
]


def activation(rng: np.random.Generator, rows: int, cols: int, n_outlier_cols: int,
               outlier_factor: float) -> np.ndarray:
    """X ~ N(0, 1) in fp32, with ``n_outlier_cols`` distinct columns (drawn from the same rng)
    multiplied by ``outlier_factor``."""
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    if n_outlier_cols:
        cols_idx = rng.choice(cols, n_outlier_cols, replace=False)
        x[:, cols_idx] *= np.float32(outlier_factor)
    return x


def weight(rng: np.random.Generator, rows: int, cols: int, std: float = 0.02) -> np.ndarray:
    return (rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)).astype(np.float32)


def grad(rng: np.random.Generator, rows: int, cols: int, std: float = 1e-3) -> np.ndarray:
    return (rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even), returned as the uint16 bit pattern.

    Done by torch (dtype plumbing, not the method): numpy has no bfloat16."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of a bf16 bit pattern to fp32 (bf16 is the top half of an fp32)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_f16(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).astype(np.float16)


# The five workloads. Sizes and distributions are those of the per-block INT8 linear layer
# benchmark set; "outliers" = (number of columns, factor).
WORKLOADS = {
    # single linear fwd, latency/correctness case
    "linear_256": dict(M=256, K=256, N=256, x_outliers=(4, 50.0), x_dtype="f32"),
    # GPT2-medium MLP fc1: tokens 4x1024, hidden 1024 -> 4096
    "gpt2m_fc1": dict(M=4096, K=1024, N=4096, x_outliers=(10, 30.0), x_dtype="bf16"),
    # hidden-4096 layer: fc1 4096 -> 16384 and fc2 16384 -> 4096 at 8192 tokens
    "h4096_fc1": dict(M=8192, K=4096, N=16384, x_outliers=(4, 50.0), x_dtype="bf16"),
    "h4096_fc2": dict(M=8192, K=16384, N=4096, x_outliers=(4, 50.0), x_dtype="bf16"),
}


def workload(name: str, seed: int = 0, *, with_grad: bool = True, with_x: bool = True):
    """Draw X [M,K], W [N,K] (and dY [M,N]) for a named GEMM workload, fp32 on the host."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(seed)
    out = {}
    if with_x:
        n_out, fac = w["x_outliers"]
        out["X"] = activation(rng, w["M"], w["K"], n_out, fac)
    out["W"] = weight(rng, w["N"], w["K"])
    if with_grad:
        out["dY"] = grad(rng, w["M"], w["N"])
    return out


def memory_sweep_input(seed: int, rows: int, cols: int = 4096) -> np.ndarray:
    """Memory-bound sweep input: N(0,1) with 1% of the channels multiplied by 100 (fp32)."""
    rng = np.random.default_rng(seed)
    return activation(rng, rows, cols, max(1, cols // 100), 100.0)


def tie_block(scale_exp: int, rng: np.random.Generator) -> np.ndarray:
    """A 32x32 fp32 block whose absmax is 127 * 2**scale_exp (so its scale is exactly
    2**scale_exp) and whose other entries are exact half-integer multiples of that scale:
    every x / s is exactly n + 0.5, the rounding tie of round-to-nearest-even."""
    s = np.float32(2.0 ** scale_exp)
    n = rng.integers(-126, 126, size=(32, 32)).astype(np.float32)
    x = (n + np.float32(0.5)) * s
    x[0, 0] = np.float32(127.0) * s
    return x.astype(np.float32)


def adversarial_blocks(seed: int = 1) -> np.ndarray:
    """A [32, 32*8] fp32 strip of eight 32x32 blocks that exercise the quantizer's edge cases:
    all-zero, a single nonzero, +-absmax ties, rounding ties, negative zeros, subnormal
    absmax (scale underflows to a subnormal), an absmax so small its scale is 0, and a
    block of identical values."""
    rng = np.random.default_rng(seed)
    b = np.zeros((32, 256), dtype=np.float32)
    # 0: all zero (left as is)
    # 1: a single nonzero
    b[7, 32 + 5] = np.float32(-3.25)
    # 2: +absmax and -absmax both present, rest Gaussian
    blk = rng.standard_normal((32, 32), dtype=np.float32)
    blk[0, 0], blk[31, 31] = np.float32(4.0), np.float32(-4.0)
    b[:, 64:96] = blk
    # 3: every x/s an exact tie
    b[:, 96:128] = tie_block(-3, rng)
    # 4: negative zeros and a few values
    blk = np.full((32, 32), -0.0, dtype=np.float32)
    blk[3, 4], blk[10, 20] = np.float32(1e-3), np.float32(-2e-3)
    b[:, 128:160] = blk
    # 5: subnormal scale: absmax 127 * 2^-140 -> s = 2^-140 (subnormal, exact)
    blk = (rng.integers(-127, 128, size=(32, 32)).astype(np.float32) * np.float32(2.0 ** -140))
    blk[0, 0] = np.float32(127.0 * 2.0 ** -140)
    b[:, 160:192] = blk
    # 6: absmax = smallest subnormal -> s = amax/127 rounds to 0 -> block quantizes to 0
    blk = np.zeros((32, 32), dtype=np.float32)
    blk[5, 5] = np.float32(2.0 ** -149)
    blk[6, 6] = -np.float32(2.0 ** -149)
    b[:, 192:224] = blk
    # 7: all entries identical
    b[:, 224:256] = np.float32(0.7)
    return b
