"""GPU parity of the forward GEMM with GELU fused into its re-quantization epilogue (f1) against the
CPU oracle: the GELU output against requant(GELU(P)) of the oracle's fp32 pre-activation P, and the
optional pre-activation output against the plain forward kernel (bit for bit)."""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import assert_requant_close, check_status, dev_qt, host

pytestmark = pytest.mark.gpu


def _operands(rows, cols, depth, rng):
    X = O.quantize_block(S.activation(rng, rows, depth, max(1, depth // 100), 30.0))
    W = O.quantize_block(S.weight(rng, cols, depth))
    return X, W


def _run(X, W, rows, cols, want_pre=True):
    Xd, Wd = dev_qt(*X), dev_qt(*W)
    Y = jf.empty_qtensor(rows, cols)
    P = jf.empty_qtensor(rows, cols) if want_pre else None
    jf.jf_linear_fwd_gelu(Xd, Wd, Y, P)
    F = jf.empty_qtensor(rows, cols)
    jf.jf_linear_fwd(Xd, Wd, F)
    out = {"y": (host(Y.q), host(Y.s)), "fwd": (host(F.q), host(F.s))}
    if want_pre:
        out["pre"] = (host(P.q), host(P.s))
    check_status()
    return out


@pytest.mark.parametrize("rows,cols,depth", [(32, 32, 32), (352, 544, 416), (256, 256, 256), (224, 1024, 1056)])
def test_fused_gelu_parity_small(rows, cols, depth):
    rng = np.random.default_rng(rows * 7 + cols * 3 + depth)
    X, W = _operands(rows, cols, depth, rng)
    out = _run(X, W, rows, cols)
    # the pre-activation output is the plain forward, from the same accumulation
    assert np.array_equal(out["pre"][0], out["fwd"][0]) and np.array_equal(out["pre"][1], out["fwd"][1])
    pre, y = O.linear_fwd_gelu(*X, *W)
    qp, sp = O.requantize(pre)
    assert_requant_close(*out["pre"], qp, sp, "pre-activation")
    qr, sr = O.requantize(y)
    assert_requant_close(*out["y"], qr, sr, "GELU output")


def test_fused_gelu_without_pre_and_hand_worked(golden_dir):
    import json, os
    g = json.load(open(os.path.join(golden_dir, "gemm_hand_64.json")))
    def const_blocks(scale, sign):
        # each block holds the constant sign * scale * 127, so its quantization scale is `scale`
        return np.kron(np.asarray(sign, np.float32) * np.asarray(scale, np.float32) * np.float32(127),
                       np.ones((32, 32), np.float32)).astype(np.float32)
    X = O.quantize_block(const_blocks(g["A_scale"], g["A_sign"]))
    W = O.quantize_block(const_blocks(g["B_scale"], g["B_sign"]))
    out = _run(X, W, 64, 64, want_pre=False)
    q, s = out["y"]
    Y = np.array(g["fwd"]["Y"], np.float32)
    pos = Y > 0
    assert np.array_equal(s[pos], np.array(g["fwd"]["s"], np.float32)[pos]) and np.all(s[~pos] == 0)
    assert np.array_equal(q, np.kron(np.where(pos, 127, 0), np.ones((32, 32))).astype(np.int8))


def test_fused_gelu_zero_depth_and_zero_blocks():
    # empty contraction: GELU(0) = 0 everywhere, pre-activation zero as well
    Xd = jf.QTensor(torch.zeros((64, 0), dtype=torch.int8, device="cuda"), torch.zeros((2, 0), device="cuda"))
    Wd = jf.QTensor(torch.zeros((96, 0), dtype=torch.int8, device="cuda"), torch.zeros((3, 0), device="cuda"))
    Y = jf.QTensor(torch.full((64, 96), 5, dtype=torch.int8, device="cuda"), torch.full((2, 3), 7.0, device="cuda"))
    P = jf.QTensor(torch.full((64, 96), 5, dtype=torch.int8, device="cuda"), torch.full((2, 3), 7.0, device="cuda"))
    jf.jf_linear_fwd_gelu(Xd, Wd, Y, P)
    assert not host(Y.q).any() and not host(Y.s).any() and not host(P.q).any() and not host(P.s).any()
    # an all-zero operand block row gives zero output blocks (scale 0)
    rng = np.random.default_rng(3)
    Xz = S.activation(rng, 96, 128, 2, 30.0)
    Xz[32:64] = 0.0
    Xq = O.quantize_block(Xz)
    Wq = O.quantize_block(S.weight(rng, 64, 128))
    out = _run(Xq, Wq, 96, 64)
    assert np.all(out["y"][1][1] == 0) and not out["y"][0][32:64].any()
    check_status()


def test_fused_gelu_workload_sampled():
    """The GPT-2-medium fc1 shape at full size: pre-activation bit-equal to the plain forward, GELU
    output on sampled blocks against the oracle."""
    d = S.workload("gpt2m_fc1", 0)
    w = S.WORKLOADS["gpt2m_fc1"]
    X = O.quantize_block(d["X"])
    W = O.quantize_block(d["W"])
    M, N = w["M"], w["N"]
    out = _run(X, W, M, N)
    assert np.array_equal(out["pre"][0], out["fwd"][0]) and np.array_equal(out["pre"][1], out["fwd"][1])
    rng = np.random.default_rng(9)
    rb = sorted(rng.choice(M // 32, 6, replace=False).tolist() + [0, M // 32 - 1])
    cb = sorted(rng.choice(N // 32, 6, replace=False).tolist() + [0, N // 32 - 1])
    pre, y = O.linear_fwd_gelu(*X, *W, rb, cb)
    ri = np.concatenate([np.arange(i * 32, i * 32 + 32) for i in rb])
    ci = np.concatenate([np.arange(j * 32, j * 32 + 32) for j in cb])
    qr, sr = O.requantize(y)
    q, s = out["y"]
    assert_requant_close(q[np.ix_(ri, ci)], s[np.ix_(rb, cb)], qr, sr, "gpt2m fc1 GELU")
