"""C ABI checks that need no GPU: the library loads, exports every function declared in
include/jetfire.h, and rejects invalid arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import int8_fully_quantized_b200 as jf
from int8_fully_quantized_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return jf.load_library()


def _declared():
    text = open(os.path.join(ROOT, "include", "jetfire.h")).read()
    return sorted(set(re.findall(r"^\s*(?:JF_API\s+)?(?:int|int64_t|const char\s*\*)\s+(jf_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("jf_quantize_block", "jf_dequantize_block", "jf_linear_fwd", "jf_linear_dgrad",
              "jf_linear_wgrad", "jf_gelu_i8", "jf_layernorm_i8", "jf_strerror", "jf_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build_lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[T]\s+(\w+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing else of the library leaks out as a C symbol
    assert sorted(n for n in exported if n.startswith("jf_")) == _declared()
    assert set(jf.EXPORTED_SYMBOLS) == set(_declared())


def test_strerror_is_total(lib):
    for st in range(-10, 2):
        assert isinstance(jf.jf_strerror(st), str) and jf.jf_strerror(st)


def test_host_validation_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)           # 16-byte aligned, never dereferenced: validation fails first
    odd = vp((1 << 20) + 4)
    # shapes must be multiples of 32
    assert lib.jf_quantize_block(fake, 1, 33, 64, fake, fake, None) == -2
    assert lib.jf_quantize_block(fake, 1, -32, 64, fake, fake, None) == -2
    # unknown dtype
    assert lib.jf_quantize_block(fake, 7, 32, 32, fake, fake, None) == -4
    # NULL pointers
    assert lib.jf_quantize_block(None, 1, 32, 32, fake, fake, None) == -1
    # misaligned codes
    assert lib.jf_quantize_block(fake, 1, 32, 32, odd, vp((1 << 21)), None) == -3
    # output overlapping the input
    assert lib.jf_quantize_block(fake, 0, 32, 32, vp((1 << 20) + 64), vp(1 << 22), None) == -5
    # empty tensors are a no-op
    assert lib.jf_quantize_block(None, 1, 0, 64, None, None, None) == 0
    # GEMM shape mismatch: X [64, 96] vs W [32, 64]
    X = jf._CQ(1 << 20, 1 << 22, 64, 96)
    W = jf._CQ(1 << 24, 1 << 26, 32, 64)
    Y = jf._Q(1 << 28, 1 << 30, 64, 32)
    assert lib.jf_linear_fwd(X, W, Y, None, None) == -2
    # GEMM output shape must be [M, N]
    W = jf._CQ(1 << 24, 1 << 26, 32, 96)
    assert lib.jf_linear_fwd(X, W, jf._Q(1 << 28, 1 << 30, 64, 64), None, None) == -2
    # no output at all
    assert lib.jf_linear_fwd(X, W, jf._Q(None, None, 64, 32), None, None) == -1
    # dgrad: dY [M, N] with W [N, K]; wgrad: dY [M, N] with X [M, K]
    assert lib.jf_linear_dgrad(jf._CQ(1 << 20, 1 << 22, 64, 96), jf._CQ(1 << 24, 1 << 26, 64, 32),
                               jf._Q(1 << 28, 1 << 30, 64, 32), None, None) == -2
    assert lib.jf_linear_wgrad(jf._CQ(1 << 20, 1 << 22, 64, 96), jf._CQ(1 << 24, 1 << 26, 96, 32),
                               jf._Q(1 << 28, 1 << 30, 96, 32), None, None) == -2
    # fused forward + GELU: the GELU output is required; the pre-activation must not alias it
    X = jf._CQ(1 << 20, 1 << 22, 64, 96)
    W = jf._CQ(1 << 24, 1 << 26, 32, 96)
    none = jf._Q(None, None, 64, 32)
    assert lib.jf_linear_fwd_gelu(X, W, none, none, None) == -1
    Y = jf._Q(1 << 28, 1 << 30, 64, 32)
    assert lib.jf_linear_fwd_gelu(X, W, Y, jf._Q((1 << 28) + 1024, 1 << 31, 64, 32), None) == -5
    assert lib.jf_linear_fwd_gelu(X, W, Y, jf._Q(1 << 31, 1 << 32, 32, 32), None) == -2
    assert lib.jf_linear_fwd_gelu(X, jf._CQ(1 << 24, 1 << 26, 32, 64), Y, none, None) == -2
    # backward of GELU: shapes must agree, dX must not alias an input
    Xc = jf._CQ(1 << 20, 1 << 22, 64, 96)
    assert lib.jf_gelu_i8_bwd(Xc, jf._CQ(1 << 24, 1 << 26, 64, 64), jf._Q(1 << 28, 1 << 30, 64, 96), None) == -2
    assert lib.jf_gelu_i8_bwd(Xc, jf._CQ(1 << 24, 1 << 26, 64, 96), jf._Q((1 << 24) + 32, 1 << 30, 64, 96),
                              None) == -5
    # backward of LayerNorm: workspace size, presence and alignment
    need = lib.jf_layernorm_i8_bwd_workspace_bytes(64, 96)
    assert need == 2 * 2 * 96 * 4 and lib.jf_layernorm_i8_bwd_workspace_bytes(33, 96) == -1
    dYc = jf._CQ(1 << 24, 1 << 26, 64, 96)
    dXq = jf._Q(1 << 28, 1 << 30, 64, 96)
    g, dg, db, ws = vp(1 << 32), vp(1 << 33), vp(1 << 34), vp(1 << 35)
    f = ctypes.c_float(1e-5)
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, g, f, dXq, dg, db, None, 0, None) == -9
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, g, f, dXq, dg, db, ws, need - 4, None) == -9
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, g, f, dXq, dg, db, vp((1 << 35) + 4), need, None) == -9
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, None, f, dXq, dg, db, ws, need, None) == -1
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, g, f, dXq, dg, vp((1 << 33) + 8), ws, need, None) == -5
    assert lib.jf_layernorm_i8_bwd(Xc, dYc, g, f, dXq, dg, db, vp((1 << 34) + 16), need, None) == -5
    # the allocation-free backward refuses shapes whose column sums exceed its 16 MiB static scratch,
    # but only after the argument checks of the workspace version (same errors, same order)
    R, H = 9472, 7104                      # 296 CTAs x 2 x 7104 x 4 bytes = 16.04 MiB, just above the limit
    assert lib.jf_layernorm_i8_bwd_workspace_bytes(R, H) == 296 * 2 * H * 4 > 16 << 20
    Xb, dYb = jf._CQ(1 << 36, 1 << 37, R, H), jf._CQ(1 << 38, 1 << 39, R, H)
    dXb = jf._Q(1 << 40, 1 << 41, R, H)
    gb, dgb, dbb = vp(1 << 42), vp(1 << 43), vp(1 << 44)
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, gb, f, dXb, dgb, dbb, None) == -9
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, gb, f, jf._Q(None, 1 << 41, R, H), dgb, dbb, None) == -1
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, jf._CQ(1 << 38, 1 << 39, R, H - 32), gb, f, dXb, dgb, dbb, None) == -2
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, vp((1 << 42) + 4), f, dXb, dgb, dbb, None) == -3
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, None, f, dXb, dgb, dbb, None) == -1
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, gb, f, jf._Q(1 << 36, 1 << 41, R, H), dgb, dbb, None) == -5
    # without dgamma and dbeta there is no scratch, so no size limit other than H <= 24576
    assert lib.jf_layernorm_i8_bwd_noalloc(Xb, dYb, gb, f, jf._Q(None, 1 << 41, R, H), None, None, None) == -1
    # granularity variants: unknown granularity, scale counts
    assert lib.jf_quantize_granular(fake, 1, 32, 64, 7, fake, fake, None) == -10
    assert [lib.jf_granular_scale_count(64, 96, g) for g in range(4)] == [6, 64, 96, 1]
    assert lib.jf_granular_scale_count(64, 96, 9) == -1
    assert lib.jf_quantization_error(fake, 1, fake, fake, 32, 32, 1, None, None) == -1
    assert lib.jf_dequantize_granular(fake, fake, 32, 32, 2, vp(1 << 20), 1, None) == -5
    # LayerNorm needs gamma/beta
    assert lib.jf_layernorm_i8(jf._CQ(1 << 20, 1 << 22, 32, 64), None, fake, ctypes.c_float(1e-5),
                               jf._Q(1 << 28, 1 << 30, 32, 64), None) == -1
    # f1 row statistics: the stats buffer is required, 8-byte aligned and apart from the other buffers
    assert lib.jf_quantize_block_rowstats(fake, 1, 32, 64, vp(1 << 22), vp(1 << 23), None, None) == -1
    assert lib.jf_quantize_block_rowstats(fake, 1, 32, 64, vp(1 << 22), vp(1 << 23), vp((1 << 24) + 4), None) == -3
    assert lib.jf_quantize_block_rowstats(fake, 1, 32, 64, vp(1 << 22), vp(1 << 23), vp((1 << 22) + 8), None) == -5
    assert lib.jf_quantize_block_rowstats(fake, 1, 33, 64, vp(1 << 22), vp(1 << 23), vp(1 << 24), None) == -2
    assert lib.jf_quantize_block_rowstats(None, 1, 0, 64, None, None, None, None) == 0
    Xl, Yl = jf._CQ(1 << 20, 1 << 22, 32, 64), jf._Q(1 << 28, 1 << 30, 32, 64)
    assert lib.jf_layernorm_i8_rowstats(Xl, None, fake, fake, ctypes.c_float(1e-5), Yl, None) == -1
    assert lib.jf_layernorm_i8_rowstats(Xl, vp((1 << 24) + 4), fake, fake, ctypes.c_float(1e-5), Yl, None) == -3
    assert lib.jf_layernorm_i8_rowstats(Xl, vp((1 << 28) + 16), fake, fake, ctypes.c_float(1e-5), Yl, None) == -5


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU behaviour")
def test_compute_without_gpu_fails_loudly(lib):
    vp = ctypes.c_void_p
    # valid arguments, but no sm_100 device is current: the call must refuse, never fall back
    st = lib.jf_quantize_block(vp(1 << 20), 1, 32, 32, vp(1 << 24), vp(1 << 26), None)
    assert st == -8
    # the allocation-free LayerNorm backward at the largest shape its static scratch takes
    # (296 x 2 x 7072 x 4 bytes = 15.97 MiB) passes every host check and stops only at the device
    R, H = 9472, 7072
    assert lib.jf_layernorm_i8_bwd_workspace_bytes(R, H) <= 16 << 20
    assert lib.jf_layernorm_i8_bwd_noalloc(jf._CQ(1 << 36, 1 << 37, R, H), jf._CQ(1 << 38, 1 << 39, R, H),
                                           vp(1 << 42), ctypes.c_float(1e-5), jf._Q(1 << 40, 1 << 41, R, H),
                                           vp(1 << 43), vp(1 << 44), None) == -8
    with pytest.raises(jf.JetfireError):
        jf._check(st, "jf_quantize_block")


def test_nvtx_instrumented_entry_points_compile(tmp_path):
    """The instrumented variant (NVTX ranges around every compute entry point, -DJF_NVTX) compiles;
    its ranges cover the same entry points the header declares."""
    src = os.path.join(build_lib.CSRC, "api.cu")
    with open(src) as f:
        text = f.read()
    assert text.count("JF_RANGE(__func__);") >= 20
    cmd = [build_lib._nvcc(), *build_lib.ARCH_FLAGS, "-O1", "-std=c++17", "-Xcompiler", "-fPIC",
           "--expt-relaxed-constexpr", "-DJF_NVTX", "-I", build_lib.INCLUDE, "-I", build_lib.CSRC, "-c", src,
           "-o", str(tmp_path / "api_nvtx.o")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
