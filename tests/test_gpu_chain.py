"""INT8 data flow between the operators of a layer (Jetfire summary, "Approach": every operator reads
and writes INT8 blocks), checked stage by stage on the GPU:

* the hidden-4096 MLP block, M = 8192: LayerNorm_i8 -> fc1 (4096 -> 16384) -> GELU_i8 -> fc2
  (16384 -> 4096), each stage run on the previous stage's GPU output; the oracle of each stage
  consumes that same GPU INT8 intermediate, so an error is attributed to the stage that made it;
* the single-linear workload end to end: fp32 X and W through the GPU quantizer into the forward.
"""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import assert_gemm_f32_close, assert_requant_close, check_status, dev_f32, dev_qt, host

pytestmark = pytest.mark.gpu


def _blocks(idx):
    return np.concatenate([np.arange(i * 32, i * 32 + 32) for i in idx])


def _sample(n, rng, k):
    return sorted(set([0, n - 1] + [int(v) for v in rng.integers(0, n, k)]))


def _magnitude(A, B, rb, cb):
    """sum_kb c * sum_k |qA||qB|: the condition scale of each sampled forward output."""
    absq = lambda q: np.abs(q.astype(np.int16)).astype(np.int8)
    return O.linear_fwd(absq(A[0]), A[1], absq(B[0]), B[1], rb, cb)


def test_mlp_block_hidden4096_stagewise():
    M, H, F = 8192, 4096, 16384
    rng = np.random.default_rng(4)
    Xq = O.quantize_block(S.activation(rng, M, H, 4, 50.0))     # INT8 input blocks of X (outlier channels)
    W1 = O.quantize_block(S.weight(rng, F, H))
    W2 = O.quantize_block(S.weight(rng, H, F))
    gamma = rng.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rng.normal(0.0, 0.1, H).astype(np.float32)

    Xd, W1d, W2d = dev_qt(*Xq), dev_qt(*W1), dev_qt(*W2)
    Xn = jf.layernorm_i8(Xd, dev_f32(gamma), dev_f32(beta), 1e-5)
    Y1, y1f = jf.linear_fwd(Xn, W1d, want_f32=True)
    G = jf.gelu_i8(Y1)
    Y2, y2f = jf.linear_fwd(G, W2d, want_f32=True)
    check_status()
    xn = (host(Xn.q), host(Xn.s))
    y1 = (host(Y1.q), host(Y1.s))
    g = (host(G.q), host(G.s))
    y2 = (host(Y2.q), host(Y2.s))
    y1f, y2f = host(y1f), host(y2f)
    del Xd, W1d, W2d, Xn, Y1, G, Y2
    torch.cuda.empty_cache()

    # LayerNorm_i8: per row, so 32-row strips are independent; sampled strips of the oracle's output
    for rb in _sample(M // 32, rng, 6):
        rows = slice(rb * 32, rb * 32 + 32)
        qo, so, _ = O.layernorm_i8(Xq[0][rows], Xq[1][rb:rb + 1], gamma, beta, 1e-5)
        assert_requant_close(xn[0][rows], xn[1][rb:rb + 1], qo, so, f"LayerNorm_i8 strip {rb}")

    # fc1 on the GPU's LayerNorm output: sampled 32x32 output blocks
    rb, cb = _sample(M // 32, rng, 6), _sample(F // 32, rng, 6)
    ref = O.linear_fwd(*xn, *W1, rb, cb)
    ri, ci = _blocks(rb), _blocks(cb)
    assert_gemm_f32_close(y1f[np.ix_(ri, ci)], ref, _magnitude(xn, W1, rb, cb), "fc1")
    qr, sr = O.quantize_block(ref)
    assert_requant_close(y1[0][np.ix_(ri, ci)], y1[1][np.ix_(rb, cb)], qr, sr, "fc1 codes")

    # GELU_i8 on the GPU's fc1 codes: the whole 8192 x 16384 tensor
    qo, so, _ = O.gelu_i8(*y1)
    assert_requant_close(g[0], g[1], qo, so, "GELU_i8 8192x16384")

    # fc2 on the GPU's GELU output (contraction 16384): sampled blocks
    rb, cb = _sample(M // 32, rng, 4), _sample(H // 32, rng, 4)
    ref = O.linear_fwd(*g, *W2, rb, cb)
    ri, ci = _blocks(rb), _blocks(cb)
    assert_gemm_f32_close(y2f[np.ix_(ri, ci)], ref, _magnitude(g, W2, rb, cb), "fc2")
    qr, sr = O.quantize_block(ref)
    assert_requant_close(y2[0][np.ix_(ri, ci)], y2[1][np.ix_(rb, cb)], qr, sr, "fc2 codes")
    # every block of both GEMMs is the quantizer rule applied to the kernel's own fp32 result
    for (q, s), f, name in ((y1, y1f, "fc1"), (y2, y2f, "fc2")):
        qq, ss = O.quantize_block(f)
        assert np.array_equal(q, qq) and np.array_equal(s, ss), name


def test_single_linear_end_to_end_from_fp32():
    """fp32 X and W (256 x 256, 4 outlier channels x50) through the GPU quantizer into the forward;
    the whole output against the oracle's quantize -> forward -> re-quantize of the same inputs."""
    d = S.workload("linear_256", 0)
    X = jf.quantize_block(dev_f32(d["X"]))
    W = jf.quantize_block(dev_f32(d["W"]))
    Y, yf = jf.linear_fwd(X, W, want_f32=True)
    check_status()
    Xr, Wr = O.quantize_block(d["X"]), O.quantize_block(d["W"])
    assert np.array_equal(host(X.q), Xr[0]) and np.array_equal(host(X.s), Xr[1])
    assert np.array_equal(host(W.q), Wr[0]) and np.array_equal(host(W.s), Wr[1])
    ref = O.linear_fwd(*Xr, *Wr)
    absq = lambda q: np.abs(q.astype(np.int16)).astype(np.int8)
    assert_gemm_f32_close(host(yf), ref, O.linear_fwd(absq(Xr[0]), Xr[1], absq(Wr[0]), Wr[1]), "single linear")
    qr, sr = O.requantize(ref)
    assert_requant_close(host(Y.q), host(Y.s), qr, sr, "single linear codes")
