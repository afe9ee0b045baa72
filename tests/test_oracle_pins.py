"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks an oracle function against a hand-worked example (``tests/golden``), a
closed form, an invariant, an independent library routine, or brute force in exact rational
arithmetic, so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from inputs import synthetic as S


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------------
# quantizer
# ---------------------------------------------------------------------------------------------
def test_quantize_hand_worked(golden_dir):
    g = _golden(golden_dir, "quantize_hand.json")
    for case in g["cases"]:
        x = np.zeros((32, 32), np.float32)
        x[0, :len(case["x"])] = np.array(case["x"], np.float32)
        q, s = O.quantize_block(x)
        assert s.shape == (1, 1)
        assert s[0, 0] == np.float32(case["s"])
        assert q[0, :len(case["q"])].tolist() == case["q"]
        assert not q[1:].any() and not q[0, len(case["q"]):].any()


def test_quantize_error_bound_brute_force():
    rng = np.random.default_rng(3)
    x = S.activation(rng, 96, 160, 5, 40.0)
    q, s = O.quantize_block(x)
    sf = O.block_scale_grid(s).astype(np.float64)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * sf)
    # q = rint(fl(x/s)); |fl(x/s) - x/s| <= 2^-24 * 128, so |x - q s| <= s (1/2 + 2^-16)
    assert np.all(err <= sf * (0.5 + 2.0 ** -16))
    assert q.min() >= -127 and q.max() <= 127
    # every block with a nonzero absmax reaches |q| = 127
    qa = np.abs(q.astype(np.int32)).reshape(3, 32, 5, 32).max(axis=(1, 3))
    assert np.all(qa[s > 0] == 127)


def test_quantize_scale_grid_orientation():
    """Block (I, J) gets absmax 127 * 2^(I - 2J): the scale grid must be exactly 2^(I - 2J),
    which fails on any transposed or mis-reshaped block bookkeeping."""
    rng = np.random.default_rng(4)
    R, C = 4 * 32, 3 * 32
    x = (rng.uniform(-1, 1, size=(R, C))).astype(np.float32)
    expect = np.zeros((4, 3), np.float32)
    for I in range(4):
        for J in range(3):
            e = I - 2 * J
            blk = x[I * 32:(I + 1) * 32, J * 32:(J + 1) * 32]
            blk *= np.float32(2.0 ** e)
            r, c = rng.integers(0, 32, 2)
            blk[r, c] = np.float32(-127.0 * 2.0 ** e if (I + J) % 2 else 127.0 * 2.0 ** e)
            expect[I, J] = np.float32(2.0 ** e)
    q, s = O.quantize_block(x)
    assert np.array_equal(s, expect)
    for I in range(4):
        for J in range(3):
            assert np.abs(q[I * 32:(I + 1) * 32, J * 32:(J + 1) * 32]).max() == 127


def test_quantize_ties_round_half_even():
    rng = np.random.default_rng(5)
    for e in (-3, 0, 4):
        x = S.tie_block(e, rng)
        q, s = O.quantize_block(x)
        assert s[0, 0] == np.float32(2.0 ** e)
        exact = x.astype(np.float64) / 2.0 ** e           # exactly n + 0.5 (or 127 at [0,0])
        ties = np.ones_like(q, dtype=bool)
        ties[0, 0] = False
        assert np.all(np.abs(q[ties] - exact[ties]) == 0.5)
        assert np.all(q[ties] % 2 == 0)
        assert q[0, 0] == 127


def test_quantize_special_blocks():
    b = S.adversarial_blocks()
    q, s = O.quantize_block(b)
    # 0: all zero
    assert s[0, 0] == 0 and not q[:, 0:32].any()
    # 1: single nonzero -> +-127 there, zero elsewhere
    assert s[0, 1] == np.float32(np.float32(3.25) / np.float32(127))
    assert q[7, 32 + 5] == -127 and np.count_nonzero(q[:, 32:64]) == 1
    # 2: both +absmax and -absmax reach +-127
    assert q[0, 64] == 127 and q[31, 95] == -127
    # 4: -0.0 entries quantize to 0; absmax from the nonzeros
    assert s[0, 4] == np.float32(np.float32(2e-3) / np.float32(127))
    assert q[10, 128 + 20] == -127 and q[3, 128 + 4] == 64  # 1e-3 / (2e-3/127) = 63.5 -> 64 (fl)
    # 5: subnormal scale 2^-140 is exact; q = the integers the block was built from
    assert s[0, 5] == np.float32(2.0 ** -140)
    blk = b[:, 160:192].astype(np.float64) / 2.0 ** -140
    assert np.array_equal(q[:, 160:192].astype(np.float64), blk)
    # 6: absmax = 2^-149 -> s = 2^-149 / 127 underflows to 0 -> q = 0
    assert s[0, 6] == 0 and not q[:, 192:224].any()
    # 7: identical entries -> all 127
    assert np.all(q[:, 224:256] == 127)


def test_quantize_per_tensor_limit():
    """With a block as large as the tensor the quantizer is per-tensor quantization; when every
    32x32 block holds the global absmax, the per-block result must equal it bit for bit."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((64, 96)).astype(np.float32)
    g = np.float32(9.0)
    for I in range(2):
        for J in range(3):
            x[I * 32 + (I * 7 + J) % 32, J * 32 + (3 * J + 1) % 32] = g if (I + J) % 2 == 0 else -g
    qb, sb = O.quantize_block(x)
    qt, st = O.quantize(x, 64, 96)
    assert st.shape == (1, 1) and st[0, 0] == np.float32(g / np.float32(127))
    assert np.all(sb == st[0, 0])
    assert np.array_equal(qb, qt)


def test_granularity_mse_direction():
    """Jetfire summary, 'Measured effects': per-block quantization lowers the quantization error
    versus per-token quantization on activations with channel-wise outliers (a direction pin)."""
    rng = np.random.default_rng(0)
    x = S.activation(rng, 512, 1024, 10, 30.0)
    mb = O.quantization_mse(x, "block")
    mt = O.quantization_mse(x, "token")
    mT = O.quantization_mse(x, "tensor")
    assert mb < mt <= mT * 1.0000001


def quarter_offset_input(granularity, rows=64, cols=64, exp=-3, seed=9):
    """An fp32 [rows, cols] tensor whose quantization error is known by hand at one granularity.

    Every group of the granularity holds one element of magnitude exactly 127 s (s = 2**exp), so
    its scale is exactly s and that element is coded without error; every other element is
    (n + 1/4) s with an integer |n| <= 100, which the quantizer codes as n, an error of exactly s/4.
    The mean squared error is therefore (1 - n_max / (rows*cols)) * s^2 / 16, with n_max the number
    of +-127 s elements. Returns (x, expected_mse)."""
    rng = np.random.default_rng(seed)
    s = np.float32(2.0 ** exp)
    x = (rng.integers(-100, 101, size=(rows, cols)).astype(np.float32) + np.float32(0.25)) * s
    br, bc = {"block": (32, 32), "token": (1, cols), "channel": (rows, 1), "tensor": (rows, cols)}[granularity]
    for I in range(rows // br):
        for J in range(cols // bc):
            r, c = I * br + int(rng.integers(0, br)), J * bc + int(rng.integers(0, bc))
            x[r, c] = np.float32(127.0) * s * np.float32(1 if rng.integers(0, 2) else -1)
    n_max = int(np.count_nonzero(np.abs(x) == np.float32(127.0) * s))
    return x.astype(np.float32), (1.0 - n_max / x.size) * float(s) ** 2 / 16.0


@pytest.mark.parametrize("granularity", ["block", "token", "channel", "tensor"])
def test_quantization_mse_hand_worked(granularity):
    """Hand-worked value of the quantization MSE: quarter-offset codes give an error of exactly s/4
    per element (s^2/16 squared) except at each group's absmax, which is exact. A sum instead of a
    mean, an absolute instead of a squared error, or a scale taken at the wrong granularity gives
    another number."""
    x, expected = quarter_offset_input(granularity)
    assert O.quantization_mse(x, granularity) == expected
    # built for one scale per tensor, the input has blocks without a 127 s element: their scales are
    # not s, so at the 32x32 granularity the error is another number
    if granularity == "tensor":
        assert O.quantization_mse(x, "block") != expected


# ---------------------------------------------------------------------------------------------
# dtype conversions and dequantize
# ---------------------------------------------------------------------------------------------
def test_bf16_conversions_match_torch():
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0e38, -1e-40], np.float32)])
    ours = O.f32_to_bf16_bits(y)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = O.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_dequantize_hand_and_round_trip():
    q = np.zeros((32, 64), np.int8)
    q[0, :4] = [1, -2, 127, -127]
    q[5, 40] = 3
    s = np.array([[0.5, 0.25]], np.float32)
    y = O.dequantize_block(q, s)
    assert y[0, :4].tolist() == [0.5, -1.0, 63.5, -63.5] and y[5, 40] == 0.75
    assert np.count_nonzero(y) == 5
    # values that are exactly q * 2^e come back exactly
    rng = np.random.default_rng(8)
    qi = rng.integers(-127, 128, size=(64, 64)).astype(np.int8)
    qi[0, 0] = 127; qi[0, 32] = 127; qi[32, 0] = 127; qi[32, 32] = -127
    x = qi.astype(np.float32) * np.float32(2.0 ** -5)
    q2, s2 = O.quantize_block(x)
    assert np.array_equal(O.dequantize_block(q2, s2), x)
    # round trip error bound on random data
    x = S.activation(rng, 64, 64, 2, 20.0)
    q3, s3 = O.quantize_block(x)
    err = np.abs(O.dequantize_block(q3, s3).astype(np.float64) - x)
    assert np.all(err <= O.block_scale_grid(s3) * (0.5 + 2.0 ** -16) + 1e-30)
    # bf16 / f16 outputs are the round-to-nearest-even of the fp32 result
    yb = O.dequantize_block(q3, s3, "bf16")
    assert np.array_equal(yb, torch.from_numpy(O.dequantize_block(q3, s3)).to(torch.bfloat16)
                          .view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(O.dequantize_block(q3, s3, "f16"),
                          torch.from_numpy(O.dequantize_block(q3, s3)).half().numpy())


# ---------------------------------------------------------------------------------------------
# the three GEMMs
# ---------------------------------------------------------------------------------------------
def _const_blocks(scale, sign):
    scale = np.asarray(scale, np.float32)
    sign = np.asarray(sign, np.float32)
    v = np.kron(sign * scale * np.float32(127), np.ones((32, 32), np.float32)).astype(np.float32)
    return v


def test_gemm_hand_worked_64(golden_dir):
    g = _golden(golden_dir, "gemm_hand_64.json")
    A = _const_blocks(g["A_scale"], g["A_sign"])
    B = _const_blocks(g["B_scale"], g["B_sign"])
    Aq, As = O.quantize_block(A)
    Bq, Bs = O.quantize_block(B)
    assert np.array_equal(As, np.array(g["A_scale"], np.float32))
    assert np.all(np.abs(Aq) == 127)
    outs = {
        "fwd": O.linear_fwd(Aq, As, Bq, Bs),
        "dgrad": O.linear_dgrad(Aq, As, Bq, Bs),
        "wgrad": O.linear_wgrad(Aq, As, Bq, Bs),
    }
    for mode, y in outs.items():
        exp = np.kron(np.array(g[mode]["Y"], np.float32), np.ones((32, 32), np.float32))
        assert np.array_equal(y, exp), mode
        q, s = O.requantize(y)
        assert np.array_equal(s, np.array(g[mode]["s"], np.float32)), mode
        assert np.array_equal(q, np.kron(np.array(g[mode]["q_sign"]) * 127, np.ones((32, 32))).astype(np.int8)), mode


def _fp32_product(a, b):
    """fp32(a*b) from the exact rational product: a*b of two fp32 values is exact in a double,
    and one conversion to fp32 rounds it once."""
    return Fraction(float(np.float32(float(Fraction(float(a)) * Fraction(float(b))))))


@pytest.mark.parametrize("mode", ["fwd", "dgrad", "wgrad"])
def test_gemm_exact_rational_brute_force(mode):
    """Brute force with Python integers and Fractions, written from the definitions
    Y = X W^T, dX = dY W, dW = dY^T X with one fp32 scale product per 32-block of the
    contraction axis. The oracle's fp32 output must be the exact value rounded (within
    0.5 ulp plus the fp64 summation slack)."""
    rng = np.random.default_rng({"fwd": 10, "dgrad": 11, "wgrad": 12}[mode])
    m, n, k = 64, 96, 96          # output rows, output cols, contraction
    def qt(r, c):
        q = rng.integers(-127, 128, size=(r, c)).astype(np.int8)
        s = (rng.uniform(0.01, 2.0, size=(r // 32, c // 32))).astype(np.float32)
        return q, s
    if mode == "fwd":
        Aq, As = qt(m, k); Bq, Bs = qt(n, k)
        y = O.linear_fwd(Aq, As, Bq, Bs)
        a = lambda i, kk: int(Aq[i, kk]); b = lambda j, kk: int(Bq[j, kk])
        sa = lambda i, kap: As[i // 32, kap]; sb = lambda j, kap: Bs[j // 32, kap]
    elif mode == "dgrad":          # A = dY [m, k], B = W [k, n]
        Aq, As = qt(m, k); Bq, Bs = qt(k, n)
        y = O.linear_dgrad(Aq, As, Bq, Bs)
        a = lambda i, kk: int(Aq[i, kk]); b = lambda j, kk: int(Bq[kk, j])
        sa = lambda i, kap: As[i // 32, kap]; sb = lambda j, kap: Bs[kap, j // 32]
    else:                          # A = dY [k, m], B = X [k, n]
        Aq, As = qt(k, m); Bq, Bs = qt(k, n)
        y = O.linear_wgrad(Aq, As, Bq, Bs)
        a = lambda i, kk: int(Aq[kk, i]); b = lambda j, kk: int(Bq[kk, j])
        sa = lambda i, kap: As[kap, i // 32]; sb = lambda j, kap: Bs[kap, j // 32]
    assert y.shape == (m, n)
    for i in range(0, m, 7):
        for j in range(0, n, 5):
            exact = Fraction(0)
            mag = Fraction(0)
            for kap in range(k // 32):
                P = sum(a(i, kk) * b(j, kk) for kk in range(kap * 32, kap * 32 + 32))
                c = _fp32_product(sa(i, kap), sb(j, kap))
                exact += c * P
                mag += abs(c * P)
            got = Fraction(float(y[i, j]))
            ulp = Fraction(float(np.spacing(np.float32(abs(y[i, j])))))
            assert abs(got - exact) <= ulp / 2 + mag * Fraction(1, 2 ** 45), (i, j)


def test_gemm_power_of_two_scales_exact():
    """All scales equal powers of two and small integer codes: every fp32 partial sum is exact,
    so Y must equal the int64 matrix product times 2^e bit for bit."""
    rng = np.random.default_rng(13)
    M, K, N = 96, 256, 64
    Xq = rng.integers(-15, 16, size=(M, K)).astype(np.int8)
    Wq = rng.integers(-15, 16, size=(N, K)).astype(np.int8)
    Xs = np.full((M // 32, K // 32), 2.0 ** -3, np.float32)
    Ws = np.full((N // 32, K // 32), 2.0 ** -6, np.float32)
    y = O.linear_fwd(Xq, Xs, Wq, Ws)
    exact = (Xq.astype(np.int64) @ Wq.astype(np.int64).T).astype(np.float64) * 2.0 ** -9
    assert np.array_equal(y.astype(np.float64), exact)
    # per-K-block powers of two (different per block): still exact
    Xs2 = (2.0 ** rng.integers(-4, 3, size=(M // 32, K // 32))).astype(np.float32)
    y2 = O.linear_fwd(Xq, Xs2, Wq, Ws)
    ex2 = np.zeros((M, N))
    for kap in range(K // 32):
        ks = slice(kap * 32, kap * 32 + 32)
        P = Xq[:, ks].astype(np.int64) @ Wq[:, ks].astype(np.int64).T
        ex2 += P * np.repeat(Xs2[:, kap].astype(np.float64), 32)[:, None] * 2.0 ** -6
    assert np.array_equal(y2.astype(np.float64), ex2)


def test_gemm_modes_are_transposes_of_each_other():
    """dX = dY W is the forward product with W^T as the weight; dW = dY^T X is the forward
    product of dY^T and X^T. Quantized blocks are square, so transposing a quantized tensor
    transposes its codes and its scale grid. Checked bit for bit (catches index-map errors)."""
    rng = np.random.default_rng(14)
    M, N, K = 96, 64, 128
    dYq, dYs = O.quantize_block(S.grad(rng, M, N))
    Wq, Ws = O.quantize_block(S.weight(rng, N, K))
    Xq, Xs = O.quantize_block(S.activation(rng, M, K, 2, 30.0))
    assert np.array_equal(O.linear_dgrad(dYq, dYs, Wq, Ws), O.linear_fwd(dYq, dYs, Wq.T.copy(), Ws.T.copy()))
    assert np.array_equal(O.linear_wgrad(dYq, dYs, Xq, Xs),
                          O.linear_fwd(dYq.T.copy(), dYs.T.copy(), Xq.T.copy(), Xs.T.copy()))
    # against a float64 matmul of the dequantized operands, when all scales of the contraction
    # axis are equal (then the per-block rescale factors out of the sum)
    Xs1 = np.repeat(Xs[:, :1], K // 32, axis=1)
    Ws1 = np.repeat(Ws[:, :1], K // 32, axis=1)
    ref = (Xq.astype(np.float64) * np.repeat(Xs1[:, 0], 32)[:, None]) @ \
          (Wq.astype(np.float64) * np.repeat(Ws1[:, 0], 32)[:, None]).T
    y = O.linear_fwd(Xq, Xs1, Wq, Ws1)
    assert np.allclose(y, ref, rtol=2e-6, atol=1e-9 * np.abs(ref).max())


def test_gemm_sampled_blocks_equal_full():
    rng = np.random.default_rng(15)
    M, N, K = 128, 96, 64
    Xq, Xs = O.quantize_block(S.activation(rng, M, K, 1, 10.0))
    Wq, Ws = O.quantize_block(S.weight(rng, N, K))
    dYq, dYs = O.quantize_block(S.grad(rng, M, N))
    full = O.linear_fwd(Xq, Xs, Wq, Ws)
    part = O.linear_fwd(Xq, Xs, Wq, Ws, row_blocks=[3, 1], col_blocks=[2])
    assert np.array_equal(part, np.concatenate([full[96:128, 64:96], full[32:64, 64:96]]))
    full = O.linear_dgrad(dYq, dYs, Wq, Ws)
    assert np.array_equal(O.linear_dgrad(dYq, dYs, Wq, Ws, [2], [0, 1]), full[64:96, 0:64])
    full = O.linear_wgrad(dYq, dYs, Xq, Xs)
    assert np.array_equal(O.linear_wgrad(dYq, dYs, Xq, Xs, [1], [1]), full[32:64, 32:64])


# ---------------------------------------------------------------------------------------------
# GELU_i8 and LayerNorm_i8
# ---------------------------------------------------------------------------------------------
def test_gelu_table_and_identities(golden_dir):
    g = _golden(golden_dir, "normal_cdf_table.json")
    x = np.array(g["x"])
    assert np.allclose(O.gelu_f64(x), x * np.array(g["Phi"]), rtol=1e-15, atol=0)
    from scipy.stats import norm
    xs = np.linspace(-8, 8, 2001)
    assert np.allclose(O.gelu_f64(xs), xs * norm.cdf(xs), rtol=1e-13, atol=1e-300)
    # Phi(x) + Phi(-x) = 1  =>  GELU(x) - GELU(-x) = x
    assert np.allclose(O.gelu_f64(xs) - O.gelu_f64(-xs), xs, rtol=0, atol=4e-15 * 8)
    assert O.gelu_f64(np.array([0.0]))[0] == 0.0


def test_linear_fwd_gelu_hand_worked_64(golden_dir):
    """Fused forward + GELU on the hand-worked constant blocks: the large positive blocks pass
    through GELU unchanged (Phi = 1 in fp64), so their codes and scales are the forward's; the large
    negative blocks become exactly zero (s = 0, q = 0)."""
    g = _golden(golden_dir, "gemm_hand_64.json")
    Aq, As = O.quantize_block(_const_blocks(g["A_scale"], g["A_sign"]))
    Bq, Bs = O.quantize_block(_const_blocks(g["B_scale"], g["B_sign"]))
    pre, y = O.linear_fwd_gelu(Aq, As, Bq, Bs)
    Y = np.array(g["fwd"]["Y"], np.float32)
    assert np.array_equal(pre, np.kron(Y, np.ones((32, 32), np.float32)))
    q, s = O.requantize(y)
    pos = Y > 0
    assert np.array_equal(s[pos], np.array(g["fwd"]["s"], np.float32)[pos])
    assert np.all(s[~pos] == 0)
    exp_q = np.kron(np.where(pos, 127, 0), np.ones((32, 32))).astype(np.int8)
    assert np.array_equal(q, exp_q)


def test_linear_fwd_gelu_normal_cdf_table(golden_dir):
    """Pre-activations built exactly equal to the table's x (power-of-two scales, one nonzero code
    per row): the fused output must be x * Phi(x) with Phi from the printed table, which it only is
    when GELU acts on the fp32 pre-activation (after re-quantization 0.5 would become 32 * 2/127)."""
    g = _golden(golden_dir, "normal_cdf_table.json")
    x = np.array(g["x"])
    Xq = np.zeros((32, 32), np.int8)
    for i, xv in enumerate(x):
        assert float(2 * xv).is_integer()                    # x = 0.25 * code * 2 * 1.0 exactly
        Xq[i, 0] = int(2 * xv)
    Xs = np.full((1, 1), 0.25, np.float32)
    Wq = np.zeros((32, 32), np.int8)
    Wq[:, 0] = 2
    Ws = np.ones((1, 1), np.float32)
    pre, y = O.linear_fwd_gelu(Xq, Xs, Wq, Ws)
    assert np.array_equal(pre[:len(x), 0], x.astype(np.float32))
    expect = x * np.array(g["Phi"])
    assert np.allclose(y[:len(x), :].astype(np.float64), expect[:, None], rtol=2.0 ** -23, atol=0)
    assert np.all(y[len(x):] == 0)


def test_gelu_i8_special_blocks():
    # all-zero block -> zero output
    q = np.zeros((32, 64), np.int8)
    s = np.array([[0.0, 0.5]], np.float32)
    qo, so, _ = O.gelu_i8(q, s)
    assert so[0, 0] == 0 and so[0, 1] == 0 and not qo.any()
    # a block of large positive values: GELU(x) = x in fp32 (Phi(x) = 1 - 1e-23), so the block
    # re-quantizes to the same codes and (within an ulp) the same scale
    rng = np.random.default_rng(16)
    q = rng.integers(1, 128, size=(32, 32)).astype(np.int8)
    q[0, 0] = 127
    s = np.array([[0.5]], np.float32)                 # smallest value 0.5*1 ... too small; shift
    x_min = 20.0
    q = (q.astype(np.int32) // 2 + 64).astype(np.int8)   # codes 64..127
    q[0, 0] = 127
    s = np.array([[x_min / 64]], np.float32)
    qo, so, y = O.gelu_i8(q, s)
    assert np.array_equal(y, q.astype(np.float32) * s[0, 0])
    assert np.array_equal(qo, q)
    assert abs(float(so[0, 0]) - float(s[0, 0])) <= float(np.spacing(s[0, 0]))
    # negative large values map to (nearly) 0: GELU(-20) ~ -5.5e-88 -> fp32 0
    qo, so, y = O.gelu_i8(-q, s)
    assert np.all(y == 0) and so[0, 0] == 0


def test_layernorm_i8_vs_torch_and_invariants():
    rng = np.random.default_rng(17)
    M, H = 64, 256
    x = S.activation(rng, M, H, 3, 50.0)
    q, s = O.quantize_block(x)
    gamma = rng.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rng.normal(0, 0.1, H).astype(np.float32)
    qo, so, y = O.layernorm_i8(q, s, gamma, beta, 1e-5)
    xd = torch.from_numpy((q.astype(np.float32) * O.block_scale_grid(s)).astype(np.float64))
    ref = torch.nn.functional.layer_norm(xd, (H,), torch.from_numpy(gamma.astype(np.float64)),
                                         torch.from_numpy(beta.astype(np.float64)),
                                         eps=float(np.float32(1e-5))).numpy()
    assert np.all(np.abs(y.astype(np.float64) - ref) <= np.abs(ref) * 2.0 ** -23 + 1e-12)
    # requantization is the block quantizer of y
    q2, s2 = O.quantize_block(y)
    assert np.array_equal(q2, qo) and np.array_equal(s2, so)
    # gamma = 1, beta = 0: rows have mean 0 and variance 1 (up to eps)
    _, _, y1 = O.layernorm_i8(q, s, np.ones(H, np.float32), np.zeros(H, np.float32), 1e-5)
    assert np.all(np.abs(y1.astype(np.float64).mean(axis=1)) < 1e-6)
    assert np.all(np.abs(y1.astype(np.float64).var(axis=1) - 1) < 1e-4)
    # scale invariance (eps = 0): doubling every block scale (exact) leaves y unchanged
    _, _, ya = O.layernorm_i8(q, s, gamma, beta, 0.0)
    _, _, yb = O.layernorm_i8(q, s * np.float32(2), gamma, beta, 0.0)
    assert np.allclose(ya, yb, rtol=0, atol=2e-6 * np.abs(ya).max())
    # a constant row gives y = beta exactly
    qc = np.full((32, H), 5, np.int8)
    sc = np.full((1, H // 32), 0.25, np.float32)
    _, _, yc = O.layernorm_i8(qc, sc, gamma, beta, 1e-5)
    assert np.array_equal(yc, np.broadcast_to(beta, yc.shape))


# ---------------------------------------------------------------------------------------------
# f2: backward of GELU_i8 and LayerNorm_i8
# ---------------------------------------------------------------------------------------------
def test_gelu_grad_against_library_table_and_differences(golden_dir):
    from scipy.stats import norm
    xs = np.linspace(-9, 9, 3601)
    d = O.gelu_grad_f64(xs)
    # library routines for Phi and phi
    # (GELU' is O(1); in the far left tail both sides carry the cancellation of Phi + x phi)
    assert np.allclose(d, norm.cdf(xs) + xs * norm.pdf(xs), rtol=1e-13, atol=1e-16)
    # the printed normal-CDF table: GELU'(x) - x phi(x) = Phi(x)
    g = _golden(golden_dir, "normal_cdf_table.json")
    x = np.array(g["x"])
    assert np.allclose(O.gelu_grad_f64(x) - x * norm.pdf(x), np.array(g["Phi"]), rtol=1e-14, atol=0)
    # central differences of the (separately pinned) GELU: a dropped term or a sign error fails
    h = 1e-5
    fd = (O.gelu_f64(xs + h) - O.gelu_f64(xs - h)) / (2 * h)
    assert np.allclose(d, fd, rtol=0, atol=1e-9)
    assert O.gelu_grad_f64(np.array([0.0]))[0] == 0.5


def test_gelu_i8_bwd_special_blocks():
    rng = np.random.default_rng(21)
    dyq = rng.integers(-127, 128, size=(32, 96)).astype(np.int8)
    dyq[0, :] = 127
    dys = np.array([[1e-3, 2e-3, 4e-3]], np.float32)
    # x block 0: large positive (GELU' = 1 exactly in fp64), block 1: large negative (GELU' = 0),
    # block 2: all zero (GELU'(0) = 1/2, exact)
    xq = np.zeros((32, 96), np.int8)
    xq[:, :32] = rng.integers(64, 128, size=(32, 32))
    xq[:, 32:64] = -rng.integers(64, 128, size=(32, 32))
    xs = np.array([[40.0 / 64, 40.0 / 64, 0.0]], np.float32)
    q, s, dx = O.gelu_i8_bwd(xq, xs, dyq, dys)
    g = dyq.astype(np.float32) * O.block_scale_grid(dys)
    assert np.array_equal(dx[:, :32], g[:, :32])
    assert np.array_equal(q[:, :32], dyq[:, :32]) and s[0, 0] == dys[0, 0]
    assert np.all(dx[:, 32:64] == 0) and s[0, 1] == 0 and not q[:, 32:64].any()
    assert np.array_equal(dx[:, 64:], g[:, 64:] * np.float32(0.5))
    assert np.array_equal(q[:, 64:], dyq[:, 64:]) and s[0, 2] == dys[0, 2] / 2


def test_layernorm_i8_bwd_vs_torch_autograd_and_invariants():
    rng = np.random.default_rng(22)
    M, H = 96, 256
    xq, xs = O.quantize_block(S.activation(rng, M, H, 3, 50.0))
    dyq, dys = O.quantize_block(S.grad(rng, M, H))
    gamma = rng.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rng.normal(0, 0.1, H).astype(np.float32)
    eps = 1e-5
    q, s, dx, dgamma, dbeta = O.layernorm_i8_bwd(xq, xs, dyq, dys, gamma, eps)
    # the library's autograd of layer_norm in fp64, on the same dequantized inputs
    x = torch.from_numpy((xq.astype(np.float32) * O.block_scale_grid(xs)).astype(np.float64)).requires_grad_()
    gm = torch.from_numpy(gamma.astype(np.float64)).requires_grad_()
    bt = torch.from_numpy(beta.astype(np.float64)).requires_grad_()
    y = torch.nn.functional.layer_norm(x, (H,), gm, bt, eps=float(np.float32(eps)))
    dy = torch.from_numpy((dyq.astype(np.float32) * O.block_scale_grid(dys)).astype(np.float64))
    y.backward(dy)
    ref = x.grad.numpy()
    assert np.allclose(dx, ref, rtol=2.0 ** -23, atol=1e-7 * np.abs(ref).max())
    assert np.allclose(dgamma, gm.grad.numpy(), rtol=2.0 ** -23, atol=1e-9 * np.abs(gm.grad.numpy()).max())
    assert np.allclose(dbeta, bt.grad.numpy(), rtol=2.0 ** -23, atol=0)
    # requantization is the block quantizer of dx
    q2, s2 = O.quantize_block(dx)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    # dx is orthogonal to the constant row (shift invariance of LayerNorm) ...
    assert np.all(np.abs(ref.sum(1)) <= 1e-9 * np.abs(ref).sum(1))
    assert np.all(np.abs(dx.astype(np.float64).sum(1)) <= 1e-6 * np.abs(dx).sum(1))
    # ... and, with eps = 0, to xhat (scale invariance; eps > 0 breaks it by eps / (var + eps))
    _, _, dx0, _, _ = O.layernorm_i8_bwd(xq, xs, dyq, dys, gamma, 0.0)
    xd = x.detach().numpy()
    xh = (xd - xd.mean(1, keepdims=True)) / np.sqrt(xd.var(1, keepdims=True))
    dx0 = dx0.astype(np.float64)
    assert np.all(np.abs((dx0 * xh).sum(1)) <= 1e-6 * np.abs(dx0 * xh).sum(1))


# ---------------------------------------------------------------------------------------------
# f3: granularity variants
# ---------------------------------------------------------------------------------------------
def test_granularity_variants_relations_and_bounds():
    """Per-channel quantization is per-token quantization of the transpose (bit for bit); per-token
    quantization of each row alone is per-tensor quantization of that row; every group reaches
    |q| = 127 and every element meets the rounding bound |x - q s| <= s/2 (1 + 2^-22)."""
    rng = np.random.default_rng(40)
    x = S.activation(rng, 96, 160, 3, 40.0)
    x[5] = 0.0                                     # an all-zero row: s = 0, codes 0
    R, C = x.shape
    qt, st = O.quantize(x, 1, C)
    qc, sc = O.quantize(x.T.copy(), 1, R)
    qch, sch = O.quantize(x, R, 1)
    assert np.array_equal(qch, qc.T) and np.array_equal(sch.ravel(), sc.ravel())
    for r in (0, 5, 17, 95):
        q1, s1 = O.quantize(x[r:r + 1], 1, C)
        assert np.array_equal(q1[0], qt[r]) and s1[0, 0] == st[r, 0]
    assert st[5, 0] == 0 and not qt[5].any()
    for (br, bc), (q, s) in {(1, C): (qt, st), (R, 1): (qch, sch), (R, C): O.quantize(x, R, C)}.items():
        sg = O.block_scale_grid(s, br, bc).astype(np.float64)
        err = np.abs(x.astype(np.float64) - q.astype(np.float64) * sg)
        assert np.all(err <= sg / 2 * (1 + 2.0 ** -22))
        qa = np.abs(q.astype(np.int32)).reshape(R // br, br, C // bc, bc).max(axis=(1, 3))
        assert np.all((qa == 127) | (s == 0))
    # dequantize at any granularity is fp32(q) * s of the element's group
    y = O.dequantize(qt, st, 1, C)
    assert np.array_equal(y, (qt.astype(np.float32) * st.astype(np.float32)).astype(np.float32))


# ---------------------------------------------------------------------------------------------
# f4: MXFP8 comparison
# ---------------------------------------------------------------------------------------------
def _e4m3_values():
    """All finite E4M3 values from the format's definition (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits; exponent field 0 is subnormal; 0x7F / 0xFF are NaN)."""
    vals = {}
    for c in range(256):
        sgn = -1.0 if c & 0x80 else 1.0
        ef, mf = (c >> 3) & 0xF, c & 0x7
        if ef == 0xF and mf == 0x7:
            continue
        vals[c] = sgn * (mf / 8.0 * 2.0 ** -6 if ef == 0 else (1 + mf / 8.0) * 2.0 ** (ef - 7))
    return vals


def test_e4m3_encode_is_nearest_even_with_saturation():
    vals = _e4m3_values()
    pos = sorted({v for v in vals.values() if v >= 0})
    rng = np.random.default_rng(50)
    xs = np.concatenate([rng.normal(0, 30, 3000), rng.uniform(-500, 500, 1000),
                         [(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])],          # every tie
                         [-(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])], [448.0, 460.0, 1e6, -1e6, 0.0]])
    xs = xs.astype(np.float32)
    codes = O.e4m3_encode(xs)
    dec = O.e4m3_decode(codes)
    for x, c, d in zip(xs, codes, dec):
        a = min(abs(float(x)), 448.0)
        best = min(pos, key=lambda p: (abs(p - a), [k for k, v in vals.items() if v == p and k < 128][0] & 1))
        assert abs(float(d)) == best, (x, d, best)
        assert d == 0 or np.sign(d) == np.sign(x)
    assert vals[int(O.e4m3_encode(np.array([448.0], np.float32))[0])] == 448.0


def test_mx_quantize_rule_hand_and_bounds():
    # one block 1..32: amax 32 -> e = 5 - 8 = -3, elements x * 8 = 8..256; E4M3 keeps 4 significant
    # bits, so 17 * 8 = 136 (between 128 and 144, a tie) goes to 128 and 18 * 8 = 144 stays
    x = np.arange(1, 33, dtype=np.float32)[None, :]
    q, sb = O.mx_quantize(x)
    assert sb[0, 0] == 127 - 3
    y = O.mx_dequantize(q, sb)[0]
    assert y[0] == 1.0 and y[16] == 16.0 and y[17] == 18.0 and y[31] == 32.0
    assert O.e4m3_decode(q)[0, 16] == 128.0          # 17 * 8 = 136 -> 128 (tie to even)
    # random blocks: the block max decodes to [256, 448] x 2^e, elements within half an E4M3 ulp
    rng = np.random.default_rng(51)
    x = S.activation(rng, 64, 256, 3, 30.0)
    x[0, :32] = 0.0
    q, sb = O.mx_quantize(x)
    assert sb[0, 0] == 0                              # all-zero block: e = -127
    v = O.e4m3_decode(q).astype(np.float64).reshape(64, 8, 32)
    e = sb.astype(np.int64) - 127
    nz = np.abs(x.reshape(64, 8, 32)).max(axis=2) > 0
    vmax = np.abs(v).max(axis=2)
    assert np.all((vmax[nz] >= 256) & (vmax[nz] <= 448))
    scaled = np.ldexp(x.reshape(64, 8, 32).astype(np.float64), -e[..., None])
    ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(scaled), 2.0 ** -6))).astype(int) - 3)
    err = np.abs(np.clip(scaled, -448, 448) - v)
    assert np.all(err <= ulp / 2 + 1e-12)


def test_mx_linear_fwd_exact_small_integers():
    """Codes that decode to small integers and power-of-two scales: the oracle's Y equals the int64
    product times the scales exactly, and the modes of the MX GEMM compose like the INT8 one."""
    rng = np.random.default_rng(52)
    M, N, K = 64, 96, 256
    ints = lambda r, c: rng.integers(-15, 16, size=(r, c)).astype(np.float32)
    A, B = ints(M, K), ints(N, K)
    Aq, As = O.e4m3_encode(A), np.full((M, K // 32), 127 + 2, np.uint8)     # scale 2^2
    Bq, Bs = O.e4m3_encode(B), np.full((N, K // 32), 127 - 1, np.uint8)     # scale 2^-1
    assert np.array_equal(O.e4m3_decode(Aq), A) and np.array_equal(O.e4m3_decode(Bq), B)
    y = O.mx_linear_fwd(Aq, As, Bq, Bs)
    assert np.array_equal(y.astype(np.float64), (A.astype(np.int64) @ B.astype(np.int64).T) * 2.0)


def test_quantize_rowstats_hand_worked_and_invariants():
    """f1 row statistics: a hand-worked block whose scale is exactly 1 (so q = x), then invariants on
    random outlier activations (block sums add up to the row sums taken over the whole row, the
    Cauchy-Schwarz bound per block) and the moments against numpy's of x = q s."""
    x = np.zeros((32, 64), np.float32)
    for r in range(32):
        x[r, :32] = r - 16          # block (0, 0): row r constant r - 16 ...
    x[0, 5] = 127.0                 # ... except one 127, which makes s = 127 / 127 = 1
    x[:, 32:] = -3.0                # block (0, 1): all -3, absmax 3, s = 3/127, q = -127
    q, s, st = O.quantize_block_rowstats(x)
    assert s[0, 0] == 1.0 and np.array_equal(q[:, :32], x[:, :32].astype(np.int8))
    # by hand: row 0 holds 31 codes -16 and one 127; row r >= 1 holds 32 codes r - 16
    assert st[0, 0, 0] == 31 * -16 + 127 == -369 and st[0, 0, 1] == 31 * 256 + 16129 == 24065
    for r in range(1, 32):
        assert st[r, 0, 0] == 32 * (r - 16) and st[r, 0, 1] == 32 * (r - 16) ** 2
    assert np.all(st[:, 1, 0] == -127 * 32) and np.all(st[:, 1, 1] == 127 * 127 * 32)

    rng = np.random.default_rng(91)
    xr = S.activation(rng, 96, 160, 2, 50.0)
    q, s, st = O.quantize_block_rowstats(xr)
    qq, ss = O.quantize_block(xr)
    assert np.array_equal(q, qq) and np.array_equal(s, ss)
    q64 = q.astype(np.int64)
    assert np.array_equal(st[:, :, 0].sum(axis=1), q64.sum(axis=1))
    assert np.array_equal(st[:, :, 1].sum(axis=1), (q64 * q64).sum(axis=1))
    assert np.all(st[:, :, 0] ** 2 <= 32 * st[:, :, 1]) and np.all(np.abs(st[:, :, 0]) <= 32 * 127)
    mean, var = O.rowstats_moments(st, s, xr.shape[1])
    xe = q.astype(np.float64) * np.repeat(np.repeat(s.astype(np.float64), 32, axis=0), 32, axis=1)
    assert np.allclose(mean, xe.mean(axis=1), rtol=1e-12, atol=1e-15)
    assert np.allclose(var, xe.var(axis=1), rtol=1e-9, atol=1e-15)
