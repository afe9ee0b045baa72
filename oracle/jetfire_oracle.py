"""CPU oracle for the per-block (32x32) INT8 data flow of Jetfire.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` use it. It shares no code with the CUDA library (``int8_fully_quantized_b200``)
and imports nothing from it.

What it computes, and where that comes from
-------------------------------------------
Source: "Jetfire: Efficient and Accurate Transformer Pretraining with INT8 Data Flow and
Per-Block Quantization" (atlas.scime.ai summary page), section "Approach": every linear and
non-linear operator reads and writes INT8 tensors that carry one scale factor per block, the
block size is B = 32, quantization happens on-chip, and the weight gradient is also an INT8
computation with per-block scales. The "Fp8 vs int8" page gives the signed INT8 range and the
dequantization x = FP(q) * s.

The pages state no formula for the scale, no rounding mode and no accumulation order. The
readings taken here:

* square 32x32 blocks, scale s = absmax(block) / 127 in fp32 (IEEE division), no zero point;
* q = clamp(rint(x / s), -127, 127): fp32 IEEE division, then round-half-to-even; -128 is never
  produced; an all-zero block (or one whose s underflows to 0) gives s = 0 and q = 0;
* linear layers: for every 32-wide block kappa of the contraction axis the integer partial sum
  P = sum q_A * q_B is exact, it is multiplied by c = fp32(s_A * s_B) (one fp32 rounding), the
  products are summed exactly enough (fp64, each c*P exact in fp64) and rounded once to fp32;
  the fp32 result is then re-quantized per 32x32 block with the rule above;
* GELU is the exact erf form 0.5 x (1 + erf(x / sqrt 2)), evaluated as 0.5 x erfc(-x / sqrt 2)
  so that it keeps its relative accuracy for negative x; LayerNorm uses the biased variance
  over the full row of the dequantized input, eps = 1e-5 by default, fp32 gamma and beta;
  both are evaluated in fp64 and rounded once to fp32 before re-quantization.

Every function below is pinned by tests in ``tests/test_oracle_pins.py`` against hand-worked
values, closed forms, brute force in exact rational arithmetic, or independent library
routines; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
QMAX = 127

__all__ = [
    "BLOCK", "QMAX", "bf16_bits_to_f32", "f32_to_bf16_bits", "quantize", "quantize_block",
    "dequantize_block", "dequantize", "block_scale_grid", "linear_fwd", "linear_fwd_gelu", "linear_dgrad", "linear_wgrad",
    "requantize", "gelu_i8", "layernorm_i8", "gelu_f64", "quantization_mse", "gelu_grad_f64",
    "gelu_i8_bwd", "layernorm_i8_bwd", "E4M3_MAX", "e4m3_encode", "e4m3_decode", "mx_quantize",
    "mx_dequantize", "mx_linear_fwd", "quantize_block_rowstats", "rowstats_moments",
]


# --------------------------------------------------------------------------------------------
# dtype helpers (exact definitions, no method arithmetic)
# --------------------------------------------------------------------------------------------
def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 (as a uint16 bit pattern) -> fp32, exact: bf16 is the upper half of an fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 with round-to-nearest-even on the dropped 16 bits (finite inputs)."""
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


# --------------------------------------------------------------------------------------------
# a1: per-block quantization (Jetfire summary, "Approach": per-block scale factors, B = 32;
#     "Fp8 vs int8" page: INT8 range -128..127, of which +-127 is used symmetrically)
# --------------------------------------------------------------------------------------------
def quantize(x: np.ndarray, block_rows: int, block_cols: int):
    """Quantize fp32 ``x`` [R, C] with one scale per ``block_rows x block_cols`` block.

    Returns (q int8 [R, C], s fp32 [R/block_rows, C/block_cols]). With 32x32 blocks this is the
    Jetfire per-block quantizer; with (R, C) blocks it is per-tensor quantization, with (1, C)
    per-token and with (R, 1) per-channel (the summary's ablation baselines)."""
    x = np.asarray(x, dtype=np.float32)
    R, C = x.shape
    if R % block_rows or C % block_cols:
        raise ValueError(f"shape {x.shape} is not a whole number of {block_rows}x{block_cols} blocks")
    nbr, nbc = R // block_rows, C // block_cols
    xb = x.reshape(nbr, block_rows, nbc, block_cols)
    # absmax of each block: exact in fp32 (|.| and max do not round); -0.0 counts as 0
    amax = np.abs(xb).max(axis=(1, 3)) if x.size else np.zeros((nbr, nbc), np.float32)
    s = (amax.astype(np.float32) / np.float32(QMAX)).astype(np.float32)     # fp32 IEEE division
    s4 = s[:, None, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (xb / s4).astype(np.float32)                                     # fp32 IEEE division
    t = np.where(s4 == 0, np.float32(0), t)                                  # zero block -> q = 0
    q = np.clip(np.rint(t), -QMAX, QMAX).astype(np.int8)                     # round half to even
    return q.reshape(R, C), s


def quantize_block(x: np.ndarray):
    """Jetfire per-block quantizer: 32x32 blocks. Input fp32 (bf16/fp16 widened exactly first)."""
    return quantize(x, BLOCK, BLOCK)


def quantize_block_rowstats(x: np.ndarray):
    """f1, second half: the per-block quantizer that also hands LayerNorm_i8 the row statistics of
    its output (the summary, "Approach": quantization on-chip, here carried one step further so that
    LayerNorm needs no pass of its own over its input to find each row's mean and variance).

    Returns (q, s, stats) with q, s as quantize_block and stats int64 [R, C/32, 2]: for row r and
    block column J, stats[r, J] = (sum of q[r, j], sum of q[r, j]^2) over the block's 32 columns.
    With x = q * s, the row's sum is sum_J s[r/32, J] * stats[r, J, 0] and its sum of squares
    sum_J s[r/32, J]^2 * stats[r, J, 1] (exact products, as the integer sums are exact)."""
    q, s = quantize_block(x)
    R, C = q.shape
    qb = q.astype(np.int64).reshape(R, C // BLOCK, BLOCK)
    stats = np.stack([qb.sum(axis=2), (qb * qb).sum(axis=2)], axis=2)
    return q, s, stats


def rowstats_moments(stats: np.ndarray, s: np.ndarray, H: int):
    """Mean and biased variance of each row of x = q * s from quantize_block_rowstats' sums, in fp64:
    mean = sum_J s S1 / H, var = sum_J s^2 S2 / H - mean^2 (clamped at 0). Returns ([R], [R])."""
    st = np.asarray(stats, np.float64)
    sr = np.repeat(np.asarray(s, np.float64), BLOCK, axis=0)  # [R, C/32]: the scale of row r's blocks
    mean = (sr * st[:, :, 0]).sum(axis=1) / H
    var = np.maximum((sr * sr * st[:, :, 1]).sum(axis=1) / H - mean * mean, 0.0)
    return mean, var


def block_scale_grid(s: np.ndarray, block_rows: int = BLOCK, block_cols: int = BLOCK) -> np.ndarray:
    """Expand a scale grid [R/br, C/bc] to one scale per element [R, C]."""
    return np.repeat(np.repeat(np.asarray(s, np.float32), block_rows, axis=0), block_cols, axis=1)


# --------------------------------------------------------------------------------------------
# a2: dequantization x = FP(q) * s ("Fp8 vs int8" page)
# --------------------------------------------------------------------------------------------
def dequantize_block(q: np.ndarray, s: np.ndarray, out: str = "f32") -> np.ndarray:
    """y = fp32(q) * s (one fp32 rounding), then round-to-nearest-even to the output dtype.

    ``out``: "f32" (fp32 array), "bf16" (uint16 bit pattern) or "f16" (float16 array)."""
    return dequantize(q, s, BLOCK, BLOCK, out)


def dequantize(q: np.ndarray, s: np.ndarray, block_rows: int, block_cols: int, out: str = "f32") -> np.ndarray:
    """dequantize_block for any block shape (the granularity variants: (1, C) per token, (R, 1) per
    channel, (R, C) per tensor), with s [R/block_rows, C/block_cols]."""
    y = (np.asarray(q).astype(np.float32) * block_scale_grid(s, block_rows, block_cols)).astype(np.float32)
    if out == "f32":
        return y
    if out == "bf16":
        return f32_to_bf16_bits(y)
    if out == "f16":
        return y.astype(np.float16)
    raise ValueError(out)


# --------------------------------------------------------------------------------------------
# a3-a5: the three INT8 GEMMs of a linear layer with per-block scales (Jetfire summary,
#        "Approach": linear operators read/write INT8 + per-block scales; the weight gradient is
#        also computed in INT8 with per-block scales).
# --------------------------------------------------------------------------------------------
def _blockscaled_sum(a_blocks, b_blocks, c_blocks):
    """sum over contraction blocks kappa of c[kappa] * (a[kappa] @ b[kappa]^T).

    a_blocks[kappa]: int8 [m, 32]; b_blocks[kappa]: int8 [n, 32];
    c_blocks[kappa]: fp32 [m, n] (the scale product, already rounded to fp32).
    The integer partial P = a @ b^T is computed as an fp64 matmul: every term and partial sum is
    an integer of magnitude <= 32 * 127^2 < 2^53, so the result is exact. c * P is exact in fp64
    (24 + 20 significant bits). The sum over kappa is fp64 and is rounded once to fp32."""
    acc = None
    for a, b, c in zip(a_blocks, b_blocks, c_blocks):
        P = a.astype(np.float64) @ b.astype(np.float64).T
        term = c.astype(np.float64) * P
        acc = term if acc is None else acc + term
    return acc.astype(np.float32)


def _rows(blocks, n_blocks):
    return range(n_blocks) if blocks is None else list(blocks)


def linear_fwd(Xq, Xs, Wq, Ws, row_blocks=None, col_blocks=None):
    """Forward Y = X W^T. X [M, K], W [N, K] -> fp32 Y [M, N] (or the sub-grid of output blocks
    ``row_blocks x col_blocks``, returned as [len(rb)*32, len(cb)*32]).

    Y[m, n] = sum_kappa fp32(sX[m/32, kappa] * sW[n/32, kappa]) * sum_{k in kappa} Xq[m,k] Wq[n,k]."""
    M, K = Xq.shape
    N = Wq.shape[0]
    rb = _rows(row_blocks, M // BLOCK)
    cb = _rows(col_blocks, N // BLOCK)
    rows = np.concatenate([np.arange(i * BLOCK, (i + 1) * BLOCK) for i in rb]) if len(rb) else np.arange(0)
    cols = np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in cb]) if len(cb) else np.arange(0)
    a_blocks, b_blocks, c_blocks = [], [], []
    for kap in range(K // BLOCK):
        ks = slice(kap * BLOCK, (kap + 1) * BLOCK)
        a_blocks.append(Xq[rows, ks])
        b_blocks.append(Wq[cols, ks])
        sa = np.repeat(Xs[list(rb), kap], BLOCK)          # per output row
        sb = np.repeat(Ws[list(cb), kap], BLOCK)          # per output col
        c_blocks.append((sa[:, None] * sb[None, :]).astype(np.float32))
    if not a_blocks:
        return np.zeros((len(rows), len(cols)), np.float32)
    return _blockscaled_sum(a_blocks, b_blocks, c_blocks)


def linear_dgrad(dYq, dYs, Wq, Ws, row_blocks=None, col_blocks=None):
    """Input gradient dX = dY W. dY [M, N], W [N, K] -> fp32 dX [M, K].

    dX[m, k] = sum_nu fp32(sdY[m/32, nu] * sW[nu, k/32]) * sum_{n in nu} dYq[m,n] Wq[n,k]."""
    M, N = dYq.shape
    K = Wq.shape[1]
    rb = _rows(row_blocks, M // BLOCK)
    cb = _rows(col_blocks, K // BLOCK)
    rows = np.concatenate([np.arange(i * BLOCK, (i + 1) * BLOCK) for i in rb]) if len(rb) else np.arange(0)
    cols = np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in cb]) if len(cb) else np.arange(0)
    a_blocks, b_blocks, c_blocks = [], [], []
    for nu in range(N // BLOCK):
        ns = slice(nu * BLOCK, (nu + 1) * BLOCK)
        a_blocks.append(dYq[rows, ns])                    # [m, 32]
        b_blocks.append(Wq[ns][:, cols].T)                # W[n in nu, k] -> [k, 32]
        sa = np.repeat(dYs[list(rb), nu], BLOCK)
        sb = np.repeat(Ws[nu, list(cb)], BLOCK)
        c_blocks.append((sa[:, None] * sb[None, :]).astype(np.float32))
    if not a_blocks:
        return np.zeros((len(rows), len(cols)), np.float32)
    return _blockscaled_sum(a_blocks, b_blocks, c_blocks)


def linear_wgrad(dYq, dYs, Xq, Xs, row_blocks=None, col_blocks=None):
    """Weight gradient dW = dY^T X. dY [M, N], X [M, K] -> fp32 dW [N, K].

    dW[n, k] = sum_mu fp32(sdY[mu, n/32] * sX[mu, k/32]) * sum_{m in mu} dYq[m,n] Xq[m,k]."""
    M, N = dYq.shape
    K = Xq.shape[1]
    rb = _rows(row_blocks, N // BLOCK)
    cb = _rows(col_blocks, K // BLOCK)
    rows = np.concatenate([np.arange(i * BLOCK, (i + 1) * BLOCK) for i in rb]) if len(rb) else np.arange(0)
    cols = np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in cb]) if len(cb) else np.arange(0)
    a_blocks, b_blocks, c_blocks = [], [], []
    for mu in range(M // BLOCK):
        ms = slice(mu * BLOCK, (mu + 1) * BLOCK)
        a_blocks.append(dYq[ms][:, rows].T)               # dY[m in mu, n] -> [n, 32]
        b_blocks.append(Xq[ms][:, cols].T)                # X[m in mu, k]  -> [k, 32]
        sa = np.repeat(dYs[mu, list(rb)], BLOCK)
        sb = np.repeat(Xs[mu, list(cb)], BLOCK)
        c_blocks.append((sa[:, None] * sb[None, :]).astype(np.float32))
    if not a_blocks:
        return np.zeros((len(rows), len(cols)), np.float32)
    return _blockscaled_sum(a_blocks, b_blocks, c_blocks)


def requantize(y: np.ndarray):
    """On-chip re-quantization of an fp32 operator output: the per-block quantizer again."""
    return quantize_block(y)


# --------------------------------------------------------------------------------------------
# a6, a7: non-linear operators on INT8 blocks (Jetfire summary, "Approach" and "Problem": the
#         memory-bound non-linear operators also read and write INT8 + per-block scales)
# --------------------------------------------------------------------------------------------
def _erfc(x: np.ndarray) -> np.ndarray:
    from scipy.special import erfc
    return erfc(x)


def gelu_f64(x: np.ndarray) -> np.ndarray:
    """GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)) in fp64, evaluated as
    0.5 x erfc(-x / sqrt 2) (the same function; 1 + erf cancels for very negative x)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * _erfc(-x / np.sqrt(2.0))


def gelu_i8(q: np.ndarray, s: np.ndarray):
    """INT8 in -> dequantize (fp32 q*s) -> GELU in fp64 -> round to fp32 -> per-block quantize.
    Returns (q_out, s_out, y_f32)."""
    x = (np.asarray(q).astype(np.float32) * block_scale_grid(s)).astype(np.float32)
    y = gelu_f64(x).astype(np.float32)
    qo, so = quantize_block(y)
    return qo, so, y


def linear_fwd_gelu(Xq, Xs, Wq, Ws, row_blocks=None, col_blocks=None):
    """Forward with GELU fused into the re-quantization epilogue (the summary's "Approach": the
    quantization, and here the activation after fc1 as well, happens on chip, before anything is
    written). Reading: GELU acts on the fp32 pre-activation P that linear_fwd returns, not on its
    INT8 re-quantization. Returns (P, y) with y = fp32(GELU_f64(P)); requantize() gives the codes
    of both outputs."""
    pre = linear_fwd(Xq, Xs, Wq, Ws, row_blocks, col_blocks)
    return pre, gelu_f64(pre.astype(np.float64)).astype(np.float32)


def layernorm_i8(q: np.ndarray, s: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
                 eps: float = 1e-5):
    """INT8 in -> x = fp32 q*s -> per row: mean, biased variance over all H columns (fp64) ->
    y = (x - mean) / sqrt(var + eps) * gamma + beta (fp64, rounded once to fp32) -> per-block
    quantize. Returns (q_out, s_out, y_f32)."""
    x = (np.asarray(q).astype(np.float32) * block_scale_grid(s)).astype(np.float64)
    H = x.shape[1]
    mu = x.sum(axis=1, keepdims=True) / H
    var = ((x - mu) ** 2).sum(axis=1, keepdims=True) / H
    y = (x - mu) / np.sqrt(var + np.float64(np.float32(eps))) * np.asarray(gamma, np.float64)[None, :] \
        + np.asarray(beta, np.float64)[None, :]
    y = y.astype(np.float32)
    qo, so = quantize_block(y)
    return qo, so, y


# --------------------------------------------------------------------------------------------
# quantization error of a granularity (Jetfire summary, "Measured effects": per-block vs
# per-token and per-channel quantization error; "Experimental setup": quantization MSE)
# --------------------------------------------------------------------------------------------
# --------------------------------------------------------------------------------------------
# f2: INT8 backward of the non-linear operators (summary, "Approach": every linear and non-linear
#     operator reads and writes INT8 with per-block scales, the backward pass included)
# --------------------------------------------------------------------------------------------
def gelu_grad_f64(x: np.ndarray) -> np.ndarray:
    """d/dx GELU(x) = Phi(x) + x phi(x) in fp64, with Phi(x) = 0.5 erfc(-x / sqrt 2) and
    phi(x) = exp(-x^2 / 2) / sqrt(2 pi) the standard normal density."""
    x = np.asarray(x, np.float64)
    return 0.5 * _erfc(-x / np.sqrt(2.0)) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)


def gelu_i8_bwd(xq: np.ndarray, xs: np.ndarray, dyq: np.ndarray, dys: np.ndarray):
    """INT8 backward of GELU_i8. x = fp32(q * s) is the pre-activation, g = fp32(q_dy * s_dy) the
    upstream gradient; dx = fp32(g * GELU'(x)) with GELU' and the product in fp64, then the
    per-block quantizer. Returns (q_dx, s_dx, dx_f32)."""
    x = (np.asarray(xq).astype(np.float32) * block_scale_grid(xs)).astype(np.float32)
    g = (np.asarray(dyq).astype(np.float32) * block_scale_grid(dys)).astype(np.float32)
    dx = (g.astype(np.float64) * gelu_grad_f64(x)).astype(np.float32)
    q, s = quantize_block(dx)
    return q, s, dx


def layernorm_i8_bwd(xq: np.ndarray, xs: np.ndarray, dyq: np.ndarray, dys: np.ndarray,
                     gamma: np.ndarray, eps: float):
    """INT8 backward of LayerNorm_i8 (the layer y = (x - mu) rstd gamma + beta of layernorm_i8).
    x = fp32(q * s) and dy = fp32(q_dy * s_dy); per row, in fp64: mu and the biased variance over
    the H columns, rstd = 1 / sqrt(var + eps), xhat = (x - mu) rstd, g = dy gamma,
      dx = rstd (g - mean(g) - xhat mean(g xhat)),
    and over the rows dgamma = sum dy xhat, dbeta = sum dy. dx is rounded to fp32 and quantized per
    block; dgamma and dbeta are rounded to fp32. Returns (q_dx, s_dx, dx_f32, dgamma, dbeta)."""
    x = (np.asarray(xq).astype(np.float32) * block_scale_grid(xs)).astype(np.float64)
    dy = (np.asarray(dyq).astype(np.float32) * block_scale_grid(dys)).astype(np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + np.float64(np.float32(eps)))
    xhat = (x - mu) * rstd
    g = dy * np.asarray(gamma, np.float32).astype(np.float64)[None, :]
    dx = rstd * (g - g.mean(axis=1, keepdims=True) - xhat * (g * xhat).mean(axis=1, keepdims=True))
    dx32 = dx.astype(np.float32)
    q, s = quantize_block(dx32)
    return q, s, dx32, (dy * xhat).sum(axis=0).astype(np.float32), dy.sum(axis=0).astype(np.float32)


# --------------------------------------------------------------------------------------------
# f4: MXFP8 comparison (not on the path: the B200's hardware block scaling, for a side-by-side
#     measurement against the per-block INT8 GEMM). OCP Microscaling Formats (MX) v1.0: blocks of
#     32 consecutive elements along the contraction axis share one E8M0 scale X = 2^e with
#     e = floor(log2(max |x|)) - emax (emax = 8 for E4M3); elements x / X are converted to E4M3.
# --------------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp32 -> FP8 E4M3 bit patterns: round to nearest, ties to even, saturating to +-448."""
    import torch
    v = np.clip(np.asarray(v, np.float32), -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(np.ascontiguousarray(v)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 bit patterns -> exact fp32 values."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float32).numpy()


def mx_quantize(x: np.ndarray):
    """MXFP8 (E4M3 elements, E8M0 scales) along the last axis of x [R, K] (K a multiple of 32).
    Per 1x32 block: e = floor(log2(max |x|)) - 8, clamped to [-127, 127] (an all-zero block takes
    -127); elements x * 2^-e (exact) rounded to E4M3, ties to even, saturating at +-448 (values in
    [448, 512) * 2^e are clamped, as the format's rule allows). Returns (codes uint8 [R, K],
    scale bytes uint8 [R, K/32] holding e + 127)."""
    x = np.asarray(x, np.float32)
    R, K = x.shape
    xb = x.reshape(R, K // 32, 32)
    amax = np.abs(xb).max(axis=2)
    _, ex = np.frexp(amax)                               # amax = m 2^ex, m in [0.5, 1)
    e = np.where(amax > 0, ex - 1 - 8, -127).clip(-127, 127).astype(np.int64)
    scaled = np.ldexp(xb.astype(np.float64), -e[..., None]).astype(np.float32)  # exact: a power of two
    return e4m3_encode(scaled).reshape(R, K), (e + 127).astype(np.uint8)


def mx_dequantize(codes: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    """Exact values (fp64) of an MXFP8 tensor: E4M3 value times 2^(byte - 127)."""
    v = e4m3_decode(codes).astype(np.float64)
    R, K = v.shape
    return np.ldexp(v.reshape(R, K // 32, 32), (sbytes.astype(np.int64) - 127)[..., None]).reshape(R, K)


def mx_linear_fwd(Aq, As, Bq, Bs):
    """Y = A B^T for MXFP8 A [M, K], B [N, K]: every product of two E4M3 values and every power-of-two
    scale is exact in fp64, and so are the per-block sums; the fp64 total is rounded once to fp32."""
    return (mx_dequantize(Aq, As) @ mx_dequantize(Bq, Bs).T).astype(np.float32)


def quantization_mse(x: np.ndarray, granularity: str) -> float:
    """Mean squared error of quantize -> dequantize for one granularity:
    "block" (32x32), "token" (one scale per row), "channel" (per column), "tensor"."""
    x = np.asarray(x, np.float32)
    R, C = x.shape
    br, bc = {"block": (BLOCK, BLOCK), "token": (1, C), "channel": (R, 1), "tensor": (R, C)}[granularity]
    q, s = quantize(x, br, bc)
    xr = q.astype(np.float32).astype(np.float64) * block_scale_grid(s, br, bc).astype(np.float64)
    return float(np.mean((xr - x.astype(np.float64)) ** 2))
