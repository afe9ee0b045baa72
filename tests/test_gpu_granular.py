"""GPU parity of the granularity variants (f3): per-token, per-channel and per-tensor quantization
and dequantization (bit-exact against the oracle for fp32, bf16 and fp16 inputs), the quantization
error sums, and the direction of the summary's ablation measured on the GPU."""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import check_status, dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu

GRAN = ["token", "channel", "tensor"]


def _block_shape(g, R, C):
    return {"block": (32, 32), "token": (1, C), "channel": (R, 1), "tensor": (R, C)}[g]


def _device_input(x32, dtype):
    """The same values on both sides: the oracle quantizes the (exactly widened) device values."""
    if dtype == "f32":
        return dev_f32(x32), x32
    if dtype == "bf16":
        bits = S.to_bf16_bits(x32)
        return dev_bf16(bits), O.bf16_bits_to_f32(bits)
    h = x32.astype(np.float16)
    return torch.from_numpy(h).cuda(), h.astype(np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("g", GRAN)
@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 160), (224, 1056), (544, 96)])
def test_granular_quantize_dequantize_bit_exact(dtype, g, rows, cols):
    rng = np.random.default_rng(rows * 3 + cols + len(g))
    x32 = S.activation(rng, rows, cols, max(1, cols // 100), 30.0)
    x32[3, :] = 0.0
    x32[:, 7] = 0.0
    xd, xh = _device_input(x32, dtype)
    q, s = jf.quantize_granular(xd, g)
    br, bc = _block_shape(g, rows, cols)
    qr, sr = O.quantize(xh, br, bc)
    assert np.array_equal(host(q), qr), f"{dtype} {g} codes"
    assert np.array_equal(host(s), sr.ravel()), f"{dtype} {g} scales"
    for out in ("f32", "bf16", "f16"):
        tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[out]
        y = torch.empty((rows, cols), dtype=tdt, device="cuda")
        jf.jf_dequantize_granular(q, s, jf.GRANULARITY[g], y)
        exp = O.dequantize(qr, sr, br, bc, out)
        got = host(y.view(torch.int16)).view(np.uint16) if out == "bf16" else host(y)
        assert np.array_equal(got.view(np.uint8), np.ascontiguousarray(exp).view(np.uint8)), f"{dtype} {g} -> {out}"
    check_status()


@pytest.mark.parametrize("g", ["block"] + GRAN)
def test_quantization_error_sums(g):
    rng = np.random.default_rng(41)
    rows, cols = 256, 1024
    x32 = S.activation(rng, rows, cols, 10, 30.0)
    xd, xh = _device_input(x32, "bf16")
    q, s = jf.quantize_granular(xd, g)
    sums = torch.empty(3, dtype=torch.float64, device="cuda")
    jf.jf_quantization_error(xd, q, s, jf.GRANULARITY[g], sums)
    got = host(sums)
    assert got[2] == got[0] / x32.size     # the MSE is the first sum over the element count
    br, bc = _block_shape(g, rows, cols)
    qr, sr = O.quantize(xh, br, bc)
    xr = qr.astype(np.float64) * O.block_scale_grid(sr, br, bc).astype(np.float64)
    sse = float(np.sum((xh.astype(np.float64) - xr) ** 2))
    assert abs(got[0] - sse) <= 1e-12 * sse
    assert abs(got[1] - float(np.sum(xh.astype(np.float64) ** 2))) <= 1e-12 * got[1]
    assert abs(got[0] / x32.size - O.quantization_mse(xh, g)) <= 1e-12 * got[0] / x32.size
    check_status()


def test_ablation_direction_on_the_gpu():
    """Per-block scales lower the error on activations with channel outliers, against per-token and
    per-tensor scales (the direction of the summary's measured effects), at the GPT2-medium fc1
    activation size."""
    d = S.workload("gpt2m_fc1", 0)
    xd = dev_bf16(S.to_bf16_bits(d["X"]))
    mse = {g: jf.quantization_mse(xd, g) for g in ["block", "token", "channel", "tensor"]}
    assert mse["block"] < mse["token"] <= mse["tensor"]
    check_status()


@pytest.mark.parametrize("g", ["block"] + GRAN)
def test_quantization_mse_hand_worked_on_the_gpu(g):
    """The hand-worked quarter-offset input (every non-absmax element coded with an error of exactly
    s/4): the GPU's MSE must equal (1 - n_max / n) s^2 / 16 exactly, since every term and partial sum
    is a multiple of 2^-10 well inside fp64."""
    from test_oracle_pins import quarter_offset_input
    x, expected = quarter_offset_input(g)
    xd = torch.from_numpy(x).cuda()
    assert jf.quantization_mse(xd, g) == expected
    check_status()
