"""GPU parity of the memory-bound per-block kernels against the CPU oracle:
quantize (a1), dequantize (a2), GELU_i8 (a6), LayerNorm_i8 (a7)."""
import zlib

import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import (assert_requant_close, check_status, dev_bf16, dev_f32, dev_qt, host)

pytestmark = pytest.mark.gpu


def _quant_gpu(x_dev):
    t = jf.quantize_block(x_dev)
    return host(t.q), host(t.s)


QUANT_SHAPES = [(32, 32), (96, 160), (256, 256), (64, 4096), (544, 96)]
ROWSTATS_SHAPES = [(32, 32), (96, 160), (64, 4096), (544, 96)]
DTYPES = ["f32", "bf16", "f16"]


def _device_input(x, dtype):
    if dtype == "f32":
        return dev_f32(x), x
    if dtype == "bf16":
        bits = S.to_bf16_bits(x)
        return dev_bf16(bits), O.bf16_bits_to_f32(bits)
    h = S.to_f16(x)
    return torch.from_numpy(h).cuda(), h.astype(np.float32)


def check_quantize(shape, dtype):
    rng = np.random.default_rng(zlib.crc32(f"{shape} {dtype}".encode()))  # stable across processes
    x = S.activation(rng, shape[0], shape[1], max(1, shape[1] // 100), 100.0)
    xd, xh = _device_input(x, dtype)
    q, s = _quant_gpu(xd)
    qr, sr = O.quantize_block(xh)
    check_status()
    assert np.array_equal(s, sr), f"{shape} {dtype}"
    assert np.array_equal(q, qr), f"{shape} {dtype}"


@pytest.mark.parametrize("shape", QUANT_SHAPES)
@pytest.mark.parametrize("dtype", DTYPES)
def test_quantize_bit_exact(shape, dtype):
    """The TMA-staged quantizer (the default kernel), including odd block-column counts (the last
    tile's second block lies past the last column)."""
    check_quantize(shape, dtype)


def test_quantize_plain_load_kernel():
    """The plain-load quantizer kernel, which the library selects for every call when JF_PLAIN_LOADS=1
    is in the environment as it loads: a child process with that setting runs the bit-exactness cases
    of both quantizer entry points (codes, scales and row statistics)."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = ("import sys; sys.path[:0] = [%r, %r]\n"
            "import test_gpu_blockwise as T\n"
            "for shp in T.QUANT_SHAPES:\n"
            "    for dt in T.DTYPES: T.check_quantize(shp, dt)\n"
            "for shp in T.ROWSTATS_SHAPES:\n"
            "    for dt in T.DTYPES: T.check_rowstats(shp, dt)\n"
            "print('plain-load cases ok')\n") % (here, os.path.dirname(here))
    res = subprocess.run([sys.executable, "-c", code], env={**os.environ, "JF_PLAIN_LOADS": "1"},
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "plain-load cases ok" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]


def test_quantize_adversarial_and_ties():
    b = S.adversarial_blocks()
    rng = np.random.default_rng(21)
    ties = np.concatenate([S.tie_block(e, rng) for e in (-20, -3, 0, 5, 30)], axis=1)
    ties = np.concatenate([ties, np.zeros((32, 96), np.float32)], axis=1)
    x = np.concatenate([b, ties], axis=0)
    q, s = _quant_gpu(dev_f32(x))
    qr, sr = O.quantize_block(x)
    check_status()
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(q, qr)


def test_quantize_random_scales_dense_ties():
    """Many blocks whose absmax spans the exponent range and whose values sit on or next to
    rounding ties of x / s."""
    rng = np.random.default_rng(22)
    R, C = 512, 512
    x = np.empty((R, C), np.float32)
    for I in range(R // 32):
        for J in range(C // 32):
            e = int(rng.integers(-60, 60))
            s = np.float32(2.0 ** e) * np.float32(rng.uniform(1, 2))
            n = rng.integers(-127, 127, size=(32, 32)).astype(np.float32) + np.float32(0.5)
            blk = (n * s).astype(np.float32)
            # nudge some entries by one ulp either way
            k = rng.integers(0, 3, size=(32, 32))
            blk = np.where(k == 1, np.nextafter(blk, np.float32(np.inf)), blk)
            blk = np.where(k == 2, np.nextafter(blk, np.float32(-np.inf)), blk)
            blk[0, 0] = np.float32(127) * s
            x[I * 32:(I + 1) * 32, J * 32:(J + 1) * 32] = blk
    q, s = _quant_gpu(dev_f32(x))
    qr, sr = O.quantize_block(x)
    check_status()
    assert np.array_equal(s, sr) and np.array_equal(q, qr)


@pytest.mark.parametrize("M", [1024, 8192])
def test_quantize_memory_sweep_full(M):
    x = S.memory_sweep_input(0, M)
    bits = S.to_bf16_bits(x)
    q, s = _quant_gpu(dev_bf16(bits))
    qr, sr = O.quantize_block(O.bf16_bits_to_f32(bits))
    check_status()
    assert np.array_equal(s, sr) and np.array_equal(q, qr)


def test_quantize_memory_sweep_65536_sampled():
    M = 65536
    x = S.memory_sweep_input(0, M)
    bits = S.to_bf16_bits(x)
    del x
    t = jf.quantize_block(dev_bf16(bits))
    q, s = host(t.q), host(t.s)
    check_status()
    xf = O.bf16_bits_to_f32
    for r0 in (0, 32768, M - 1024):
        qr, sr = O.quantize_block(xf(bits[r0:r0 + 1024]))
        assert np.array_equal(q[r0:r0 + 1024], qr) and np.array_equal(s[r0 // 32:(r0 + 1024) // 32], sr)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_dequantize_bit_exact(dtype):
    rng = np.random.default_rng(23)
    x = S.activation(rng, 160, 288, 3, 60.0)
    x[:32, :32] = 0.0
    qr, sr = O.quantize_block(x)
    t = dev_qt(qr, sr)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    y = jf.dequantize_block(t, tdt)
    torch.cuda.synchronize()
    ref = O.dequantize_block(qr, sr, dtype)
    check_status()
    if dtype == "bf16":
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    elif dtype == "f16":
        assert np.array_equal(y.cpu().numpy().view(np.uint16), ref.view(np.uint16))
    else:
        assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_dequantize_memory_sweep_bf16():
    x = S.memory_sweep_input(1, 8192)
    qr, sr = O.quantize_block(x)
    y = jf.dequantize_block(dev_qt(qr, sr), torch.bfloat16)
    ref = O.dequantize_block(qr, sr, "bf16")
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    check_status()


@pytest.mark.parametrize("shape", [(32, 32), (96, 160), (256, 1024)])
def test_gelu_i8(shape):
    rng = np.random.default_rng(24)
    x = S.activation(rng, shape[0], shape[1], max(1, shape[1] // 100), 30.0)
    qr, sr = O.quantize_block(x)
    y = jf.gelu_i8(dev_qt(qr, sr))
    q, s = host(y.q), host(y.s)
    check_status()
    qo, so, _ = O.gelu_i8(qr, sr)
    assert_requant_close(q, s, qo, so, "gelu_i8")


def test_gelu_i8_special_blocks():
    # zero block, large positive block, large negative block, tiny scale block
    rng = np.random.default_rng(25)
    q = np.zeros((32, 128), np.int8)
    q[:, 32:64] = rng.integers(64, 128, size=(32, 32))
    q[:, 64:96] = -rng.integers(64, 128, size=(32, 32))
    q[:, 96:128] = rng.integers(-127, 128, size=(32, 32))
    s = np.array([[0.0, 0.3, 0.3, 1e-30]], np.float32)
    y = jf.gelu_i8(dev_qt(q, s))
    qg, sg = host(y.q), host(y.s)
    qo, so, _ = O.gelu_i8(q, s)
    check_status()
    assert_requant_close(qg, sg, qo, so, "gelu special")
    assert sg[0, 0] == 0 and not qg[:, :32].any()


def test_gelu_i8_negative_tail_relative_accuracy():
    """A block whose values are all <= -3: GELU is small there and the block scale follows it;
    the erfc form keeps the relative accuracy the scale needs."""
    rng = np.random.default_rng(26)
    q = -rng.integers(100, 128, size=(64, 64)).astype(np.int8)
    s = np.full((2, 2), np.float32(5.0 / 127), np.float32)
    y = jf.gelu_i8(dev_qt(q, s))
    qo, so, _ = O.gelu_i8(q, s)
    assert_requant_close(host(y.q), host(y.s), qo, so, "gelu tail")


@pytest.mark.parametrize("M,H", [(32, 32), (64, 1024), (96, 4096), (32, 6144)])
def test_layernorm_i8(M, H):
    rng = np.random.default_rng(27)
    x = S.activation(rng, M, H, max(1, H // 100), 50.0)
    qr, sr = O.quantize_block(x)
    gamma = rng.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rng.normal(0, 0.2, H).astype(np.float32)
    y = jf.layernorm_i8(dev_qt(qr, sr), dev_f32(gamma), dev_f32(beta), 1e-5)
    qg, sg = host(y.q), host(y.s)
    check_status()
    qo, so, _ = O.layernorm_i8(qr, sr, gamma, beta, 1e-5)
    assert_requant_close(qg, sg, qo, so, "layernorm_i8")


def test_layernorm_i8_constant_rows():
    H = 256
    q = np.full((64, H), 7, np.int8)
    s = np.full((2, H // 32), 0.5, np.float32)
    gamma = np.linspace(0.5, 2, H).astype(np.float32)
    beta = np.linspace(-1, 1, H).astype(np.float32)
    y = jf.layernorm_i8(dev_qt(q, s), dev_f32(gamma), dev_f32(beta), 1e-5)
    qo, so, yo = O.layernorm_i8(q, s, gamma, beta, 1e-5)
    assert np.array_equal(yo, np.broadcast_to(beta, yo.shape))
    assert_requant_close(host(y.q), host(y.s), qo, so, "layernorm const")


def test_memory_sweep_nonlinear_8192():
    """GELU_i8 and LayerNorm_i8 at the memory-sweep size M = 8192, H = 4096."""
    x = S.memory_sweep_input(2, 8192)
    qr, sr = O.quantize_block(x)
    t = dev_qt(qr, sr)
    g = jf.gelu_i8(t)
    qo, so, _ = O.gelu_i8(qr, sr)
    assert_requant_close(host(g.q), host(g.s), qo, so, "gelu 8192")
    gamma = np.ones(4096, np.float32)
    beta = np.zeros(4096, np.float32)
    ln = jf.layernorm_i8(t, dev_f32(gamma), dev_f32(beta), 1e-5)
    qo, so, _ = O.layernorm_i8(qr, sr, gamma, beta, 1e-5)
    assert_requant_close(host(ln.q), host(ln.s), qo, so, "layernorm 8192")
    check_status()


def test_empty_inputs_are_noops():
    z = torch.empty((0, 64), device="cuda")
    t = jf.quantize_block(z)
    assert t.q.shape == (0, 64)
    check_status()


# --------------------------------------------------------------------------------------------
# f1, second half: the quantizer hands LayerNorm_i8 its row statistics
# --------------------------------------------------------------------------------------------
def check_rowstats(shape, dtype):
    rng = np.random.default_rng(zlib.crc32(f"rowstats {shape} {dtype}".encode()))
    x = S.activation(rng, shape[0], shape[1], max(1, shape[1] // 100), 60.0)
    x[5, :] = 0.0
    xd, xh = _device_input(x, dtype)
    t, st = jf.quantize_block_rowstats(xd)
    qr, sr, str_ = O.quantize_block_rowstats(xh)
    check_status()
    assert np.array_equal(host(t.q), qr) and np.array_equal(host(t.s), sr), f"{shape} {dtype}"
    assert np.array_equal(host(st).astype(np.int64), str_), f"{shape} {dtype}"


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", ROWSTATS_SHAPES)
def test_quantize_rowstats_bit_exact(shape, dtype):
    """Codes and scales equal jf_quantize_block's and the oracle's; the per-row, per-block sums of q
    and q^2 equal the oracle's exactly, on odd block-column counts too (the plain-load kernel is
    checked by test_quantize_plain_load_kernel)."""
    check_rowstats(shape, dtype)


@pytest.mark.parametrize("M,H", [(32, 32), (64, 1024), (96, 4096), (32, 6144), (8192, 4096)])
def test_layernorm_i8_from_rowstats(M, H):
    """LayerNorm_i8 with the row statistics from the quantizer against the oracle's LayerNorm_i8 of
    the same codes, and against the kernel that finds the statistics itself."""
    rng = np.random.default_rng(zlib.crc32(f"ln rowstats {M} {H}".encode()))
    x = S.activation(rng, M, H, max(1, H // 100), 50.0)
    gamma = rng.uniform(0.5, 1.5, H).astype(np.float32)
    beta = rng.normal(0, 0.2, H).astype(np.float32)
    X, st = jf.quantize_block_rowstats(dev_f32(x))
    y = jf.layernorm_i8_rowstats(X, st, dev_f32(gamma), dev_f32(beta), 1e-5)
    y_ref_gpu = jf.layernorm_i8(X, dev_f32(gamma), dev_f32(beta), 1e-5)
    check_status()
    qr, sr = O.quantize_block(x)
    assert np.array_equal(host(X.q), qr) and np.array_equal(host(X.s), sr)
    if M <= 96:
        qo, so, _ = O.layernorm_i8(qr, sr, gamma, beta, 1e-5)
        assert_requant_close(host(y.q), host(y.s), qo, so, "layernorm_i8 from row stats")
    else:  # full size: sampled strips against the oracle
        for r0 in (0, M // 2 - 32, M - 32):
            qo, so, _ = O.layernorm_i8(qr[r0:r0 + 32], sr[r0 // 32:r0 // 32 + 1], gamma, beta, 1e-5)
            assert_requant_close(host(y.q)[r0:r0 + 32], host(y.s)[r0 // 32:r0 // 32 + 1], qo, so, "sampled strip")
    assert_requant_close(host(y.q), host(y.s), host(y_ref_gpu.q), host(y_ref_gpu.s), "from stats vs own pass")
