"""GPU parity of the INT8 backward of GELU_i8 and LayerNorm_i8 (f2) against the CPU oracle: the
re-quantized input gradients to within the stated LSB tolerance, dgamma and dbeta to 1e-5 of their
condition scale, from one block up to the hidden-4096 sizes."""
import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import GEMM_RTOL, assert_requant_close, check_status, dev_f32, dev_qt, host

pytestmark = pytest.mark.gpu


def _pair(rng, rows, cols, spread=1.0):
    X = O.quantize_block(S.activation(rng, rows, cols, max(1, cols // 100), 30.0) * spread)
    dY = O.quantize_block(S.grad(rng, rows, cols))
    return X, dY


def _gelu_bwd_gpu(X, dY, rows, cols):
    dX = jf.empty_qtensor(rows, cols)
    jf.jf_gelu_i8_bwd(dev_qt(*X), dev_qt(*dY), dX)
    q, s = host(dX.q), host(dX.s)
    check_status()
    return q, s


@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 160), (224, 1056), (512, 512)])
def test_gelu_bwd_parity(rows, cols):
    rng = np.random.default_rng(rows + 3 * cols)
    X, dY = _pair(rng, rows, cols)
    q, s = _gelu_bwd_gpu(X, dY, rows, cols)
    qr, sr, _ = O.gelu_i8_bwd(*X, *dY)
    assert_requant_close(q, s, qr, sr, f"gelu bwd {rows}x{cols}")


def test_gelu_bwd_special_blocks():
    rng = np.random.default_rng(31)
    dyq = rng.integers(-127, 128, size=(32, 128)).astype(np.int8)
    dyq[0, :] = 127
    dys = np.array([[1e-3, 2e-3, 4e-3, 8e-3]], np.float32)
    xq = np.zeros((32, 128), np.int8)
    xq[:, :32] = rng.integers(64, 128, size=(32, 32))        # GELU' = 1
    xq[:, 32:64] = -rng.integers(64, 128, size=(32, 32))     # GELU' = 0
    xq[:, 96:] = rng.integers(-127, 128, size=(32, 32))     # ordinary block
    xs = np.array([[40.0 / 64, 40.0 / 64, 0.0, 0.05]], np.float32)  # block 2 all zero: GELU' = 1/2
    q, s = _gelu_bwd_gpu((xq, xs), (dyq, dys), 32, 128)
    qr, sr, _ = O.gelu_i8_bwd(xq, xs, dyq, dys)
    assert np.array_equal(q[:, :96], qr[:, :96]) and np.array_equal(s[:, :3], sr[:, :3])
    assert np.array_equal(q[:, :32], dyq[:, :32]) and not q[:, 32:64].any() and s[0, 1] == 0
    assert_requant_close(q, s, qr, sr, "gelu bwd special")


def test_gelu_bwd_hidden4096_sampled():
    """The fc1 activation size of the hidden-4096 layer (8192 x 16384), oracle on sampled blocks."""
    rows, cols = 8192, 16384
    rng = np.random.default_rng(32)
    X, dY = _pair(rng, rows, cols)
    q, s = _gelu_bwd_gpu(X, dY, rows, cols)
    for bi, bj in [(0, 0), (rows // 32 - 1, cols // 32 - 1)] + [tuple(x) for x in rng.integers(0, [rows // 32, cols // 32], size=(30, 2))]:
        rs, cs = slice(bi * 32, bi * 32 + 32), slice(bj * 32, bj * 32 + 32)
        qr, sr, _ = O.gelu_i8_bwd(X[0][rs, cs], X[1][bi:bi + 1, bj:bj + 1], dY[0][rs, cs], dY[1][bi:bi + 1, bj:bj + 1])
        assert_requant_close(q[rs, cs], s[bi:bi + 1, bj:bj + 1], qr, sr, f"block {bi},{bj}")


def _ln_bwd_gpu(X, dY, gamma, eps, want_params=True):
    rows, cols = X[0].shape
    dX = jf.empty_qtensor(rows, cols)
    g = dev_f32(gamma)
    dg = torch.empty(cols, dtype=torch.float32, device="cuda") if want_params else None
    db = torch.empty(cols, dtype=torch.float32, device="cuda") if want_params else None
    ws = None
    if want_params:
        ws = torch.full((jf.jf_layernorm_i8_bwd_workspace_bytes(rows, cols),), 0x7F, dtype=torch.uint8, device="cuda")
    jf.jf_layernorm_i8_bwd(dev_qt(*X), dev_qt(*dY), g, eps, dX, dg, db, ws)
    out = (host(dX.q), host(dX.s), host(dg) if want_params else None, host(db) if want_params else None)
    check_status()
    return out


def _assert_param_grad_close(got, ref, mag, what):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= GEMM_RTOL * mag), f"{what}: worst {(err / np.maximum(mag, 1e-300)).max():.2e}"


def _ln_terms(X, dY, gamma, eps):
    """Condition scales of dgamma and dbeta: sum over rows of |dy xhat| and |dy| (fp64)."""
    x = (X[0].astype(np.float32) * O.block_scale_grid(X[1])).astype(np.float64)
    dy = (dY[0].astype(np.float32) * O.block_scale_grid(dY[1])).astype(np.float64)
    xh = (x - x.mean(1, keepdims=True)) / np.sqrt(x.var(1, keepdims=True) + np.float32(eps))
    return np.abs(dy * xh).sum(0), np.abs(dy).sum(0)


@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 256), (64, 1056), (256, 4096)])
def test_layernorm_bwd_parity(rows, cols):
    rng = np.random.default_rng(7 * rows + cols)
    X, dY = _pair(rng, rows, cols)
    gamma = rng.uniform(0.5, 1.5, cols).astype(np.float32)
    eps = 1e-5
    q, s, dg, db = _ln_bwd_gpu(X, dY, gamma, eps)
    qr, sr, _, dgr, dbr = O.layernorm_i8_bwd(*X, *dY, gamma, eps)
    assert_requant_close(q, s, qr, sr, f"ln bwd dX {rows}x{cols}")
    mg, mb = _ln_terms(X, dY, gamma, eps)
    _assert_param_grad_close(dg, dgr, mg, "dgamma")
    _assert_param_grad_close(db, dbr, mb, "dbeta")
    # deterministic: a second call gives the same bits
    q2, s2, dg2, db2 = _ln_bwd_gpu(X, dY, gamma, eps)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    assert np.array_equal(dg.view(np.uint32), dg2.view(np.uint32)) and np.array_equal(db.view(np.uint32), db2.view(np.uint32))
    # without parameter gradients no workspace is needed, and dX is unchanged
    q3, s3, _, _ = _ln_bwd_gpu(X, dY, gamma, eps, want_params=False)
    assert np.array_equal(q, q3) and np.array_equal(s, s3)


def test_layernorm_bwd_constant_rows_and_zero_gradient():
    rng = np.random.default_rng(33)
    cols = 256
    xq = np.full((64, cols), 5, np.int8)                     # constant rows: xhat = 0
    xs = np.full((2, cols // 32), 0.25, np.float32)
    dyq, dys = O.quantize_block(S.grad(rng, 64, cols))
    dyq[32:] = 0                                              # second strip: zero upstream gradient
    dys[1] = 0
    gamma = rng.uniform(0.5, 1.5, cols).astype(np.float32)
    q, s, dg, db = _ln_bwd_gpu((xq, xs), (dyq, dys), gamma, 1e-5)
    qr, sr, _, dgr, dbr = O.layernorm_i8_bwd(xq, xs, dyq, dys, gamma, 1e-5)
    assert_requant_close(q, s, qr, sr, "constant rows")
    assert not q[32:].any() and np.all(s[1] == 0)
    assert np.all(dg == 0)                                    # dy * xhat with xhat = 0
    _assert_param_grad_close(db, dbr, np.abs(dyq.astype(np.float64) * O.block_scale_grid(dys)).sum(0), "dbeta")


def test_layernorm_bwd_hidden4096_full():
    """The LayerNorm size of the hidden-4096 layer (8192 x 4096): dX on sampled strips, dgamma and
    dbeta over all rows (oracle evaluated per 1024-row chunk, partial sums added in fp64)."""
    rows, cols = 8192, 4096
    rng = np.random.default_rng(34)
    X, dY = _pair(rng, rows, cols)
    gamma = rng.uniform(0.5, 1.5, cols).astype(np.float32)
    eps = 1e-5
    q, s, dg, db = _ln_bwd_gpu(X, dY, gamma, eps)
    dgr = np.zeros(cols)
    dbr = np.zeros(cols)
    mg = np.zeros(cols)
    mb = np.zeros(cols)
    for r0 in range(0, rows, 1024):
        rs, bs = slice(r0, r0 + 1024), slice(r0 // 32, (r0 + 1024) // 32)
        Xc, dYc = (X[0][rs], X[1][bs]), (dY[0][rs], dY[1][bs])
        qr, sr, _, g_, b_ = O.layernorm_i8_bwd(*Xc, *dYc, gamma, eps)
        dgr += g_
        dbr += b_
        a, b = _ln_terms(Xc, dYc, gamma, eps)
        mg += a
        mb += b
        if r0 in (0, rows - 1024, 4096):
            assert_requant_close(q[rs], s[bs], qr, sr, f"dX rows {r0}..")
    # the chunked oracle carries its own fp32 rounding per chunk: allow it on top of the tolerance
    _assert_param_grad_close(dg, dgr, mg + 8 * np.abs(dgr) * 2.0 ** -24 / GEMM_RTOL, "dgamma")
    _assert_param_grad_close(db, dbr, mb + 8 * np.abs(dbr) * 2.0 ** -24 / GEMM_RTOL, "dbeta")
