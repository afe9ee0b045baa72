"""GPU parity of the MXFP8 comparison path (f4): MX quantization bit-exact against the oracle, and the
block-scaled tensor-core GEMM against the oracle's exact products."""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import check_status, dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu


def _dev(x32, dtype):
    if dtype == "f32":
        return dev_f32(x32), x32
    if dtype == "bf16":
        bits = S.to_bf16_bits(x32)
        return dev_bf16(bits), O.bf16_bits_to_f32(bits)
    h = x32.astype(np.float16)
    return torch.from_numpy(h).cuda(), h.astype(np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 160), (256, 1024)])
def test_mx_quantize_bit_exact(dtype, rows, cols):
    rng = np.random.default_rng(rows + cols)
    x32 = S.activation(rng, rows, cols, max(1, cols // 100), 30.0)
    x32[1, :32] = 0.0
    x32[2, 32:64] = 1e-30 if dtype == "f32" else 0.0
    xd, xh = _dev(x32, dtype)
    q, s = jf.mx_quantize(xd)
    qr, sr = O.mx_quantize(xh)
    assert np.array_equal(host(s), sr), "scale bytes"
    assert np.array_equal(host(q), qr), "codes"
    check_status()


def test_mx_gemm_exact_integers_and_scales():
    """Codes that decode to small integers and per-block power-of-two scales that differ per row, per
    column and per K block: every product and partial sum is exact in fp32, so Y must equal the
    oracle bit for bit (a wrong scale-factor layout in TMEM shows up here)."""
    rng = np.random.default_rng(60)
    M, N, K = 256, 384, 512
    A = rng.integers(-15, 16, size=(M, K)).astype(np.float32)
    B = rng.integers(-15, 16, size=(N, K)).astype(np.float32)
    Aq, Bq = O.e4m3_encode(A), O.e4m3_encode(B)
    As = (127 + rng.integers(-3, 4, size=(M, K // 32))).astype(np.uint8)
    Bs = (127 + rng.integers(-3, 4, size=(N, K // 32))).astype(np.uint8)
    yr = O.mx_linear_fwd(Aq, As, Bq, Bs)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y = host(jf.mx_linear_fwd(d(Aq), d(As), d(Bq), d(Bs)))
    assert np.array_equal(y, yr)
    check_status()


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (224, 160, 1024), (4096, 4096, 1024)])
def test_mx_gemm_vs_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    X = S.to_bf16_bits(S.activation(rng, M, K, max(1, K // 100), 30.0))
    W = S.to_bf16_bits(S.weight(rng, N, K))
    Xd, Wd = dev_bf16(X), dev_bf16(W)
    Aq, As = jf.mx_quantize(Xd)
    Bq, Bs = jf.mx_quantize(Wd)
    y = host(jf.mx_linear_fwd(Aq, As, Bq, Bs))
    aq, as_, bq, bs = host(Aq), host(As), host(Bq), host(Bs)
    if M * N > 1 << 20:     # full size: sampled 128-row / 128-column strips
        ri = np.r_[0:128, M - 128:M]
        ci = np.r_[0:128, N - 128:N]
        yr = O.mx_linear_fwd(aq[ri], as_[ri], bq[ci], bs[ci])
        mag = np.abs(O.mx_dequantize(aq[ri], as_[ri])) @ np.abs(O.mx_dequantize(bq[ci], bs[ci])).T
        y = y[np.ix_(ri, ci)]
    else:
        yr = O.mx_linear_fwd(aq, as_, bq, bs)
        mag = np.abs(O.mx_dequantize(aq, as_)) @ np.abs(O.mx_dequantize(bq, bs)).T
    err = np.abs(y.astype(np.float64) - yr.astype(np.float64))
    assert np.all(err <= 1e-5 * mag + 1e-30), f"worst {(err / np.maximum(mag, 1e-30)).max():.2e}"
    assert np.linalg.norm(err) <= 1e-5 * np.linalg.norm(yr)
    check_status()
