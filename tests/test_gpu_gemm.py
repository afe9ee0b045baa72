"""GPU parity of the block-scaled INT8 GEMMs (forward a3, input gradient a4, weight gradient a5)
against the CPU oracle, from single blocks with ragged tiles up to the full workload sizes."""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import assert_gemm_f32_close, assert_requant_close, check_status, dev_qt, host

pytestmark = pytest.mark.gpu

ORACLE = {"fwd": O.linear_fwd, "dgrad": O.linear_dgrad, "wgrad": O.linear_wgrad}
GPU = {"fwd": jf.jf_linear_fwd, "dgrad": jf.jf_linear_dgrad, "wgrad": jf.jf_linear_wgrad}


def _operands(mode, rows, cols, depth, rng):
    """Quantized operands (host) of the GEMM whose output is [rows, cols] with contraction depth."""
    if mode == "fwd":      # X [rows, depth], W [cols, depth]
        A = O.quantize_block(S.activation(rng, rows, depth, max(1, depth // 100), 30.0))
        B = O.quantize_block(S.weight(rng, cols, depth))
    elif mode == "dgrad":  # dY [rows, depth], W [depth, cols]
        A = O.quantize_block(S.grad(rng, rows, depth))
        B = O.quantize_block(S.weight(rng, depth, cols))
    else:                  # dY [depth, rows], X [depth, cols]
        A = O.quantize_block(S.grad(rng, depth, rows))
        B = O.quantize_block(S.activation(rng, depth, cols, max(1, cols // 100), 30.0))
    return A, B


def _magnitude(mode, A, B, rb=None, cb=None):
    """sum_kb c * sum_k |qA||qB| >= sum_kb |c P|: the condition scale of each output."""
    return ORACLE[mode](np.abs(A[0].astype(np.int16)).astype(np.int8), A[1],
                        np.abs(B[0].astype(np.int16)).astype(np.int8), B[1], rb, cb)


def _run_gpu(mode, A, B, rows, cols):
    Ad, Bd = dev_qt(*A), dev_qt(*B)
    Y = jf.empty_qtensor(rows, cols)
    yf = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    GPU[mode](Ad, Bd, Y, yf)
    q, s, y = host(Y.q), host(Y.s), host(yf)
    check_status()
    return q, s, y


SHAPES = [
    (32, 32, 32),      # one block, partial tile in every direction
    (128, 256, 128),   # exactly one tile, one stage
    (352, 544, 416),   # 3 x 3 tiles with ragged edges, 13 contraction blocks (ragged stage)
    (256, 256, 256),   # the single-linear workload
    (224, 1024, 1056),
    (544, 352, 416),   # more rows than columns: the column tiles vary fastest
    (1056, 224, 96),   # the same with three contraction blocks (one partial stage)
]


@pytest.mark.parametrize("mode", ["fwd", "dgrad", "wgrad"])
@pytest.mark.parametrize("rows,cols,depth", SHAPES)
def test_gemm_parity_small(mode, rows, cols, depth):
    rng = np.random.default_rng(rows * 7 + cols * 3 + depth + {"fwd": 0, "dgrad": 1, "wgrad": 2}[mode])
    A, B = _operands(mode, rows, cols, depth, rng)
    q, s, y = _run_gpu(mode, A, B, rows, cols)
    y_ref = ORACLE[mode](*A, *B)
    assert_gemm_f32_close(y, y_ref, _magnitude(mode, A, B), mode)
    # the on-chip re-quantization applies the quantizer rule to the kernel's own fp32 result
    qq, ss = O.quantize_block(y)
    assert np.array_equal(s, ss) and np.array_equal(q, qq)
    qr, sr = O.requantize(y_ref)
    assert_requant_close(q, s, qr, sr, mode)


@pytest.mark.parametrize("mode", ["fwd", "dgrad", "wgrad"])
def test_gemm_hand_worked_64(mode, golden_dir):
    import json, os
    g = json.load(open(os.path.join(golden_dir, "gemm_hand_64.json")))
    const = lambda sc, sg: np.kron(np.asarray(sg, np.float32) * np.asarray(sc, np.float32) * np.float32(127),
                                   np.ones((32, 32), np.float32)).astype(np.float32)
    A = O.quantize_block(const(g["A_scale"], g["A_sign"]))
    B = O.quantize_block(const(g["B_scale"], g["B_sign"]))
    q, s, y = _run_gpu(mode, A, B, 64, 64)
    assert np.array_equal(y, np.kron(np.array(g[mode]["Y"], np.float32), np.ones((32, 32), np.float32)))
    assert np.array_equal(s, np.array(g[mode]["s"], np.float32))
    assert np.array_equal(q, np.kron(np.array(g[mode]["q_sign"]) * 127, np.ones((32, 32))).astype(np.int8))


def test_gemm_power_of_two_exact():
    """Power-of-two scales and small codes: every fp32 partial sum is exact in any order, so the
    GPU result must equal the int64 product times the scale bit for bit."""
    rng = np.random.default_rng(31)
    M, K, N = 384, 1024, 512
    Xq = rng.integers(-15, 16, size=(M, K)).astype(np.int8)
    Wq = rng.integers(-15, 16, size=(N, K)).astype(np.int8)
    Xs = np.full((M // 32, K // 32), 2.0 ** -3, np.float32)
    Ws = np.full((N // 32, K // 32), 2.0 ** -7, np.float32)
    q, s, y = _run_gpu("fwd", (Xq, Xs), (Wq, Ws), M, N)
    exact = (Xq.astype(np.int64) @ Wq.astype(np.int64).T).astype(np.float64) * 2.0 ** -10
    assert np.array_equal(y.astype(np.float64), exact)


def test_gemm_zero_blocks_and_zero_depth():
    rng = np.random.default_rng(32)
    A, B = _operands("fwd", 128, 256, 128, rng)
    Aq = A[0].copy(); As = A[1].copy()
    Aq[:32] = 0; As[0] = 0                  # a whole row block of zeros -> zero output blocks
    q, s, y = _run_gpu("fwd", (Aq, As), B, 128, 256)
    assert not y[:32].any() and not q[:32].any() and not s[0].any()
    # contraction length 0: exact zeros
    Y = jf.empty_qtensor(64, 64)
    yf = torch.full((64, 64), 7.0, device="cuda")
    e = jf.QTensor(torch.empty((64, 0), dtype=torch.int8, device="cuda"),
                   torch.empty((2, 0), dtype=torch.float32, device="cuda"))
    jf.jf_linear_fwd(e, e, Y, yf)
    assert not host(yf).any() and not host(Y.q).any() and not host(Y.s).any()
    check_status()


def test_gemm_codes_only_and_f32_only_outputs():
    rng = np.random.default_rng(33)
    A, B = _operands("dgrad", 256, 512, 384, rng)
    Ad, Bd = dev_qt(*A), dev_qt(*B)
    Y = jf.empty_qtensor(256, 512)
    jf.jf_linear_dgrad(Ad, Bd, Y, None)
    yf = torch.empty((256, 512), dtype=torch.float32, device="cuda")
    jf.jf_linear_dgrad(Ad, Bd, None, yf)
    q, s, y = host(Y.q), host(Y.s), host(yf)
    qq, ss = O.quantize_block(y)
    assert np.array_equal(q, qq) and np.array_equal(s, ss)
    check_status()


# ----------------------------------------------------------------- full workload sizes
def _sample_blocks(n_rb, n_cb, rng, k=24):
    rb = sorted(set([0, n_rb - 1] + list(rng.integers(0, n_rb, k // 2))))
    cb = sorted(set([0, n_cb - 1] + list(rng.integers(0, n_cb, k // 2))))
    return rb, cb


def _full_size_case(name, mode, seed=0):
    w = S.WORKLOADS[name]
    d = S.workload(name, seed)
    Xq, Xs = O.quantize_block(d["X"])
    Wq, Ws = O.quantize_block(d["W"])
    dYq, dYs = O.quantize_block(d["dY"])
    M, K, N = w["M"], w["K"], w["N"]
    if mode == "fwd":
        return (Xq, Xs), (Wq, Ws), M, N
    if mode == "dgrad":
        return (dYq, dYs), (Wq, Ws), M, K
    return (dYq, dYs), (Xq, Xs), N, K


@pytest.mark.parametrize("mode", ["fwd", "dgrad", "wgrad"])
@pytest.mark.parametrize("name", ["linear_256", "gpt2m_fc1"])
def test_gemm_workloads_sampled(name, mode):
    A, B, rows, cols = _full_size_case(name, mode)
    q, s, y = _run_gpu(mode, A, B, rows, cols)
    qq, ss = O.quantize_block(y)
    assert np.array_equal(q, qq) and np.array_equal(s, ss)
    rng = np.random.default_rng(5)
    rb, cb = _sample_blocks(rows // 32, cols // 32, rng)
    y_ref = ORACLE[mode](*A, *B, rb, cb)
    rows_idx = np.concatenate([np.arange(i * 32, i * 32 + 32) for i in rb])
    cols_idx = np.concatenate([np.arange(j * 32, j * 32 + 32) for j in cb])
    y_sub = y[np.ix_(rows_idx, cols_idx)]
    assert_gemm_f32_close(y_sub, y_ref, _magnitude(mode, A, B, rb, cb), f"{name} {mode}")
    qr, sr = O.quantize_block(y_ref)
    assert_requant_close(q[np.ix_(rows_idx, cols_idx)], s[np.ix_(rb, cb)], qr, sr, f"{name} {mode}")


@pytest.mark.parametrize("mode", ["fwd", "dgrad", "wgrad"])
@pytest.mark.parametrize("name", ["h4096_fc1", "h4096_fc2"])
def test_gemm_hidden4096_sampled(name, mode):
    A, B, rows, cols = _full_size_case(name, mode)
    q, s, y = _run_gpu(mode, A, B, rows, cols)
    rng = np.random.default_rng(6)
    rb, cb = _sample_blocks(rows // 32, cols // 32, rng, k=12)
    y_ref = ORACLE[mode](*A, *B, rb, cb)
    rows_idx = np.concatenate([np.arange(i * 32, i * 32 + 32) for i in rb])
    cols_idx = np.concatenate([np.arange(j * 32, j * 32 + 32) for j in cb])
    assert_gemm_f32_close(y[np.ix_(rows_idx, cols_idx)], y_ref, _magnitude(mode, A, B, rb, cb), f"{name} {mode}")
    qr, sr = O.quantize_block(y_ref)
    assert_requant_close(q[np.ix_(rows_idx, cols_idx)], s[np.ix_(rb, cb)], qr, sr, f"{name} {mode}")
    # the re-quantization of every block is the quantizer rule applied to the fp32 result
    qq, ss = O.quantize_block(y)
    assert np.array_equal(q, qq) and np.array_equal(s, ss)


# ----------------------------------------------------------------- plain INT8 product (tensor ceiling)
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (384, 512, 1024), (256, 768, 4096)])
def test_plain_int8_gemm_exact(M, N, K):
    """jf_gemm_i8_s32, the unscaled INT8 product the bench uses as the measured tensor-core
    ceiling: exact against the int64 product, including the extreme codes -128 and 127."""
    rng = np.random.default_rng(M + N + K)
    a = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    b = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    a[0, :] = -128
    b[0, :] = -128
    b[1, :] = 127
    c = torch.empty((M, N), dtype=torch.int32, device="cuda")
    jf.jf_gemm_i8_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), c)
    ref = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(host(c).astype(np.int64), ref)
    check_status()
