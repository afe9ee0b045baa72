"""Helpers shared by the GPU parity tests (host <-> device marshalling and the tolerances)."""
import numpy as np
import torch

import int8_fully_quantized_b200 as jf
import oracle as O

DEV = "cuda"

# Tolerances (stated once, used by every parity test):
#  * quantize / dequantize: bit-exact codes, scales and outputs;
#  * fp32 GEMM outputs: per element |y - y_ref| <= 1e-5 * sum_kb c*|qA||qB| (the condition scale of
#    the sum) and ||y - y_ref||_2 <= 1e-5 ||y_ref||_2;
#  * re-quantized outputs (GEMM, GELU_i8, LayerNorm_i8): |q - q_ref| <= 1 everywhere, at most 0.1% of
#    the codes differ, block scales within 1e-5 relative.
GEMM_RTOL = 1e-5
MAX_LSB_FRACTION = 1e-3
SCALE_RTOL = 1e-5


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def dev_qt(q, s):
    return jf.QTensor(torch.from_numpy(np.ascontiguousarray(q, dtype=np.int8)).to(DEV),
                      torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).to(DEV))


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check_status():
    assert jf.jf_device_status() == 0


def assert_requant_close(q, s, q_ref, s_ref, what=""):
    q = np.asarray(q, np.int32)
    q_ref = np.asarray(q_ref, np.int32)
    d = np.abs(q - q_ref)
    assert d.max(initial=0) <= 1, f"{what}: code differs by {d.max()}"
    frac = np.count_nonzero(d) / max(1, d.size)
    assert frac <= MAX_LSB_FRACTION, f"{what}: {frac:.2e} of the codes differ by 1 LSB"
    s = np.asarray(s, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    assert np.all(np.abs(s - s_ref) <= SCALE_RTOL * s_ref), f"{what}: scale off by {np.max(np.abs(s - s_ref) / np.maximum(s_ref, 1e-300)):.2e}"
    return frac


def assert_gemm_f32_close(y, y_ref, mag, what=""):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    err = np.abs(y - y_ref)
    bad = err > GEMM_RTOL * np.asarray(mag, np.float64)
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond 1e-5 of their condition scale; worst {(err / np.maximum(mag, 1e-300)).max():.2e}"
    nr = np.linalg.norm(y_ref)
    assert np.linalg.norm(y - y_ref) <= GEMM_RTOL * nr + 1e-300, f"{what}: normwise {np.linalg.norm(y - y_ref) / nr:.2e}"
