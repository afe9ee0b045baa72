"""GPU checks of jf_layernorm_i8_bwd_noalloc, the allocation-free variant of the LayerNorm backward
whose per-CTA column sums live in the library's static device scratch: it must give the same bits
as the workspace version, agree with the oracle, and refuse shapes whose sums do not fit."""
import ctypes

import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import GEMM_RTOL, assert_requant_close, check_status, dev_f32, dev_qt, host

pytestmark = pytest.mark.gpu


def _inputs(rows, cols, seed):
    rng = np.random.default_rng(seed)
    X = O.quantize_block(S.activation(rng, rows, cols, max(1, cols // 100), 30.0))
    dY = O.quantize_block(S.grad(rng, rows, cols))
    gamma = rng.uniform(0.5, 1.5, cols).astype(np.float32)
    return X, dY, gamma


# (9472, 7072) needs 296 x 2 x 7072 x 4 bytes = 15.97 MiB, the top of the 16 MiB static scratch, so the
# last CTAs' column sums sit at its very end.
@pytest.mark.parametrize("rows,cols", [(96, 256), (8192, 4096), (9472, 7072)])
def test_noalloc_matches_workspace_version_and_oracle(rows, cols):
    X, dY, gamma = _inputs(rows, cols, rows + cols)
    Xd, dYd, g = dev_qt(*X), dev_qt(*dY), dev_f32(gamma)
    outs = []
    for variant in ("workspace", "noalloc", "noalloc"):
        dX = jf.empty_qtensor(rows, cols)
        dg = torch.empty(cols, dtype=torch.float32, device="cuda")
        db = torch.empty(cols, dtype=torch.float32, device="cuda")
        if variant == "workspace":
            ws = torch.empty(jf.jf_layernorm_i8_bwd_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
            jf.jf_layernorm_i8_bwd(Xd, dYd, g, 1e-5, dX, dg, db, ws)
        else:
            jf.jf_layernorm_i8_bwd_noalloc(Xd, dYd, g, 1e-5, dX, dg, db)
        outs.append((host(dX.q), host(dX.s), host(dg), host(db)))
        check_status()
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    if rows <= 96:
        qr, sr, _, dgr, dbr = O.layernorm_i8_bwd(*X, *dY, gamma, 1e-5)
        assert_requant_close(outs[1][0], outs[1][1], qr, sr, "noalloc dX")
        x = (X[0].astype(np.float32) * O.block_scale_grid(X[1])).astype(np.float64)
        dy = (dY[0].astype(np.float32) * O.block_scale_grid(dY[1])).astype(np.float64)
        xh = (x - x.mean(1, keepdims=True)) / np.sqrt(x.var(1, keepdims=True) + np.float32(1e-5))
        assert np.all(np.abs(outs[1][2] - dgr) <= GEMM_RTOL * np.abs(dy * xh).sum(0))
        assert np.all(np.abs(outs[1][3] - dbr) <= GEMM_RTOL * np.abs(dy).sum(0))


def test_noalloc_without_parameter_gradients():
    X, dY, gamma = _inputs(64, 512, 5)
    dX = jf.empty_qtensor(64, 512)
    jf.jf_layernorm_i8_bwd_noalloc(dev_qt(*X), dev_qt(*dY), dev_f32(gamma), 1e-5, dX)
    qr, sr, _, _, _ = O.layernorm_i8_bwd(*X, *dY, gamma, 1e-5)
    assert_requant_close(host(dX.q), host(dX.s), qr, sr, "noalloc dX only")
    check_status()


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    lib = jf.load_library()
    rows, cols = 32768, 8192          # 296 CTAs x 2 x 8192 x 4 bytes = 19.4 MB > 16 MiB
    assert jf.jf_layernorm_i8_bwd_workspace_bytes(rows, cols) > 16 << 20
    X = jf.QTensor(torch.empty((rows, cols), dtype=torch.int8, device="cuda"),
                   torch.empty((rows // 32, cols // 32), device="cuda"))
    dX = jf.empty_qtensor(rows, cols)
    g = torch.ones(cols, device="cuda")
    dg, db = torch.empty(cols, device="cuda"), torch.empty(cols, device="cuda")
    st = lib.jf_layernorm_i8_bwd_noalloc(jf._cq(X), jf._cq(X), ctypes.c_void_p(g.data_ptr()), ctypes.c_float(1e-5),
                                         jf._q(dX, rows, cols), ctypes.c_void_p(dg.data_ptr()),
                                         ctypes.c_void_p(db.data_ptr()), None)
    assert st == -9
    check_status()
