"""Python binding of the per-block INT8 data-flow library (``libjetfire.so``, C ABI in
``include/jetfire.h``).

The binding only marshals arguments: tensors are torch CUDA tensors (torch provides device memory
and streams), every step of the computation runs in the library's sm_100a kernels. There is no
fallback: importing works without a GPU (so the C ABI can be inspected), but every compute call
raises if the library is missing or no B200 is current.

A quantized tensor is a pair ``QTensor(q, s)``: ``q`` int8 [rows, cols] codes and ``s`` fp32
[rows/32, cols/32] block scales, both contiguous on the device. Block (I, J) covers rows
32I..32I+31 and columns 32J..32J+31 (Jetfire summary, "Approach": per-block scales, B = 32).
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

from . import build_lib
from .build_lib import LIB_PATH

__all__ = [
    "QTensor", "JetfireError", "load_library", "empty_qtensor", "EXPORTED_SYMBOLS", "JF_F32", "JF_BF16", "JF_F16",
    "GRANULARITY",
    # C ABI, one wrapper per entry point
    "jf_quantize_block", "jf_dequantize_block", "jf_linear_fwd", "jf_linear_fwd_gelu", "jf_linear_dgrad",
    "jf_linear_wgrad", "jf_gelu_i8", "jf_layernorm_i8", "jf_gelu_i8_bwd", "jf_layernorm_i8_bwd",
    "jf_quantize_block_rowstats", "jf_layernorm_i8_rowstats", "quantize_block_rowstats", "layernorm_i8_rowstats",
    "jf_layernorm_i8_bwd_workspace_bytes", "jf_layernorm_i8_bwd_noalloc", "jf_quantize_granular",
    "jf_dequantize_granular", "jf_quantization_error", "jf_granular_scale_count", "jf_mx_quantize",
    "jf_mx_linear_fwd", "jf_gemm_i8_s32", "jf_selftest_wait_timeout", "jf_strerror",
    "jf_device_status", "jf_sm_count",
    # allocating helpers
    "quantize_block", "dequantize_block", "linear_fwd", "linear_fwd_gelu", "linear_dgrad", "linear_wgrad",
    "gelu_i8", "layernorm_i8", "gelu_i8_bwd", "layernorm_i8_bwd", "quantize_granular", "quantization_mse",
    "mx_quantize", "mx_linear_fwd",
]

JF_F32, JF_BF16, JF_F16 = 0, 1, 2
GRANULARITY = {"block": 0, "token": 1, "channel": 2, "tensor": 3}
_DTYPES = {torch.float32: JF_F32, torch.bfloat16: JF_BF16, torch.float16: JF_F16}

EXPORTED_SYMBOLS = (
    "jf_quantize_block", "jf_quantize_block_rowstats", "jf_layernorm_i8_rowstats", "jf_dequantize_block", "jf_linear_fwd", "jf_linear_fwd_gelu", "jf_linear_dgrad",
    "jf_linear_wgrad",
    "jf_gelu_i8", "jf_layernorm_i8", "jf_gelu_i8_bwd", "jf_layernorm_i8_bwd", "jf_layernorm_i8_bwd_workspace_bytes",
    "jf_layernorm_i8_bwd_noalloc", "jf_quantize_granular", "jf_dequantize_granular", "jf_quantization_error",
    "jf_granular_scale_count", "jf_mx_quantize", "jf_mx_linear_fwd", "jf_gemm_i8_s32", "jf_selftest_wait_timeout",
    "jf_strerror",
    "jf_device_status",
    "jf_sm_count",
)


class _CQ(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("s", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class _Q(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("s", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class JetfireError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {jf_strerror(status)} (status {status})")


_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libjetfire.so`` (built by ``build_lib``) once and declare its prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("JETFIRE_LIB", LIB_PATH)
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m int8_fully_quantized_b200.build_lib`")
    if path == LIB_PATH and not build_lib.up_to_date():
        raise RuntimeError(f"{path} was not built from the current sources: rebuild it with "
                           "`python -m int8_fully_quantized_b200.build_lib`")
    lib = ctypes.CDLL(path)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.jf_quantize_block.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    lib.jf_dequantize_block.argtypes = [vp, vp, i64, i64, vp, i32, vp]
    for name in ("jf_linear_fwd", "jf_linear_dgrad", "jf_linear_wgrad"):
        getattr(lib, name).argtypes = [_CQ, _CQ, _Q, vp, vp]
    lib.jf_linear_fwd_gelu.argtypes = [_CQ, _CQ, _Q, _Q, vp]
    lib.jf_gelu_i8.argtypes = [_CQ, _Q, vp]
    lib.jf_layernorm_i8.argtypes = [_CQ, vp, vp, ctypes.c_float, _Q, vp]
    lib.jf_quantize_block_rowstats.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp]
    lib.jf_layernorm_i8_rowstats.argtypes = [_CQ, vp, vp, vp, ctypes.c_float, _Q, vp]
    lib.jf_gelu_i8_bwd.argtypes = [_CQ, _CQ, _Q, vp]
    lib.jf_layernorm_i8_bwd.argtypes = [_CQ, _CQ, vp, ctypes.c_float, _Q, vp, vp, vp, i64, vp]
    lib.jf_layernorm_i8_bwd_workspace_bytes.argtypes = [i64, i64]
    lib.jf_layernorm_i8_bwd_noalloc.argtypes = [_CQ, _CQ, vp, ctypes.c_float, _Q, vp, vp, vp]
    lib.jf_quantize_granular.argtypes = [vp, i32, i64, i64, i32, vp, vp, vp]
    lib.jf_dequantize_granular.argtypes = [vp, vp, i64, i64, i32, vp, i32, vp]
    lib.jf_quantization_error.argtypes = [vp, i32, vp, vp, i64, i64, i32, vp, vp]
    lib.jf_granular_scale_count.argtypes = [i64, i64, i32]
    lib.jf_mx_quantize.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    lib.jf_mx_linear_fwd.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
    lib.jf_gemm_i8_s32.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    lib.jf_selftest_wait_timeout.argtypes = [i64, vp]
    lib.jf_strerror.argtypes = [i32]
    lib.jf_strerror.restype = ctypes.c_char_p
    lib.jf_device_status.argtypes = [vp]
    lib.jf_sm_count.argtypes = []
    for name in EXPORTED_SYMBOLS:
        if name != "jf_strerror":
            getattr(lib, name).restype = ctypes.c_int
    lib.jf_layernorm_i8_bwd_workspace_bytes.restype = i64
    lib.jf_granular_scale_count.restype = i64
    _lib = lib
    return lib


class QTensor(NamedTuple):
    q: torch.Tensor
    s: torch.Tensor

    @property
    def rows(self) -> int:
        return self.q.shape[0]

    @property
    def cols(self) -> int:
        return self.q.shape[1]


def empty_qtensor(rows: int, cols: int, device="cuda") -> QTensor:
    return QTensor(torch.empty((rows, cols), dtype=torch.int8, device=device),
                   torch.empty((rows // 32, cols // 32), dtype=torch.float32, device=device))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr() if t.numel() else None


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cq(t: QTensor) -> _CQ:
    return _CQ(_ptr(t.q), _ptr(t.s), t.q.shape[0], t.q.shape[1])


def _q(t: Optional[QTensor], rows: int, cols: int) -> _Q:
    if t is None:
        return _Q(None, None, rows, cols)
    return _Q(_ptr(t.q), _ptr(t.s), t.q.shape[0], t.q.shape[1])


def _check(status: int, where: str) -> None:
    if status != 0:
        raise JetfireError(status, where)


# --------------------------------------------------------------------------- C ABI, same names
def jf_quantize_block(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, stream=None) -> None:
    lib = load_library()
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {x.dtype}")
    _check(lib.jf_quantize_block(_ptr(x), _DTYPES[x.dtype], x.shape[0], x.shape[1], _ptr(q), _ptr(s),
                                 _stream(stream)), "jf_quantize_block")


def jf_quantize_block_rowstats(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, stats: torch.Tensor,
                               stream=None) -> None:
    lib = load_library()
    _check(lib.jf_quantize_block_rowstats(_ptr(x), _DTYPES[x.dtype], x.shape[0], x.shape[1], _ptr(q), _ptr(s),
                                          _ptr(stats), _stream(stream)), "jf_quantize_block_rowstats")


def jf_dequantize_block(q: torch.Tensor, s: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    lib = load_library()
    if y.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {y.dtype}")
    _check(lib.jf_dequantize_block(_ptr(q), _ptr(s), q.shape[0], q.shape[1], _ptr(y), _DTYPES[y.dtype],
                                   _stream(stream)), "jf_dequantize_block")


def jf_linear_fwd(X: QTensor, W: QTensor, Y: Optional[QTensor], y_f32: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    lib = load_library()
    _check(lib.jf_linear_fwd(_cq(X), _cq(W), _q(Y, X.rows, W.rows), _ptr(y_f32), _stream(stream)), "jf_linear_fwd")


def jf_linear_fwd_gelu(X: QTensor, W: QTensor, Y: QTensor, Ypre: Optional[QTensor] = None, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_linear_fwd_gelu(_cq(X), _cq(W), _q(Y, X.rows, W.rows), _q(Ypre, X.rows, W.rows), _stream(stream)),
           "jf_linear_fwd_gelu")


def jf_linear_dgrad(dY: QTensor, W: QTensor, dX: Optional[QTensor], dx_f32: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    lib = load_library()
    _check(lib.jf_linear_dgrad(_cq(dY), _cq(W), _q(dX, dY.rows, W.cols), _ptr(dx_f32), _stream(stream)),
           "jf_linear_dgrad")


def jf_linear_wgrad(dY: QTensor, X: QTensor, dW: Optional[QTensor], dw_f32: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    lib = load_library()
    _check(lib.jf_linear_wgrad(_cq(dY), _cq(X), _q(dW, dY.cols, X.cols), _ptr(dw_f32), _stream(stream)),
           "jf_linear_wgrad")


def jf_gelu_i8(X: QTensor, Y: QTensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_gelu_i8(_cq(X), _q(Y, X.rows, X.cols), _stream(stream)), "jf_gelu_i8")


def jf_layernorm_i8(X: QTensor, gamma: torch.Tensor, beta: torch.Tensor, eps: float, Y: QTensor,
                    stream=None) -> None:
    lib = load_library()
    _check(lib.jf_layernorm_i8(_cq(X), _ptr(gamma), _ptr(beta), ctypes.c_float(eps), _q(Y, X.rows, X.cols),
                               _stream(stream)), "jf_layernorm_i8")


def jf_layernorm_i8_rowstats(X: QTensor, stats: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, eps: float,
                             Y: QTensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_layernorm_i8_rowstats(_cq(X), _ptr(stats), _ptr(gamma), _ptr(beta), ctypes.c_float(eps),
                                        _q(Y, X.rows, X.cols), _stream(stream)), "jf_layernorm_i8_rowstats")


def jf_gelu_i8_bwd(X: QTensor, dY: QTensor, dX: QTensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_gelu_i8_bwd(_cq(X), _cq(dY), _q(dX, X.rows, X.cols), _stream(stream)), "jf_gelu_i8_bwd")


def jf_layernorm_i8_bwd_workspace_bytes(rows: int, cols: int) -> int:
    return int(load_library().jf_layernorm_i8_bwd_workspace_bytes(rows, cols))


def jf_layernorm_i8_bwd(X: QTensor, dY: QTensor, gamma: torch.Tensor, eps: float, dX: QTensor,
                        dgamma: Optional[torch.Tensor] = None, dbeta: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load_library()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.jf_layernorm_i8_bwd(_cq(X), _cq(dY), _ptr(gamma), ctypes.c_float(eps), _q(dX, X.rows, X.cols),
                                   _ptr(dgamma), _ptr(dbeta), _ptr(workspace), nbytes, _stream(stream)),
           "jf_layernorm_i8_bwd")


def jf_layernorm_i8_bwd_noalloc(X: QTensor, dY: QTensor, gamma: torch.Tensor, eps: float, dX: QTensor,
                                dgamma: Optional[torch.Tensor] = None, dbeta: Optional[torch.Tensor] = None,
                                stream=None) -> None:
    lib = load_library()
    _check(lib.jf_layernorm_i8_bwd_noalloc(_cq(X), _cq(dY), _ptr(gamma), ctypes.c_float(eps), _q(dX, X.rows, X.cols),
                                           _ptr(dgamma), _ptr(dbeta), _stream(stream)), "jf_layernorm_i8_bwd_noalloc")


def jf_granular_scale_count(rows: int, cols: int, g: int) -> int:
    return int(load_library().jf_granular_scale_count(rows, cols, g))


def jf_quantize_granular(x: torch.Tensor, g: int, q: torch.Tensor, s: torch.Tensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_quantize_granular(_ptr(x), _DTYPES[x.dtype], x.shape[0], x.shape[1], g, _ptr(q), _ptr(s),
                                    _stream(stream)), "jf_quantize_granular")


def jf_dequantize_granular(q: torch.Tensor, s: torch.Tensor, g: int, y: torch.Tensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_dequantize_granular(_ptr(q), _ptr(s), q.shape[0], q.shape[1], g, _ptr(y), _DTYPES[y.dtype],
                                      _stream(stream)), "jf_dequantize_granular")


def jf_quantization_error(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: int, sums: torch.Tensor,
                          stream=None) -> None:
    lib = load_library()
    _check(lib.jf_quantization_error(_ptr(x), _DTYPES[x.dtype], _ptr(q), _ptr(s), x.shape[0], x.shape[1], g,
                                     _ptr(sums), _stream(stream)), "jf_quantization_error")


def quantize_granular(x: torch.Tensor, granularity: str, stream=None):
    """(codes, scales) of x at one granularity: "block", "token", "channel" or "tensor"."""
    g = GRANULARITY[granularity]
    q = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    s = torch.empty(jf_granular_scale_count(x.shape[0], x.shape[1], g), dtype=torch.float32, device=x.device)
    jf_quantize_granular(x, g, q, s, stream)
    return q, s


def quantization_mse(x: torch.Tensor, granularity: str, stream=None) -> float:
    """Mean squared error of quantize -> dequantize at one granularity, computed on the GPU."""
    q, s = quantize_granular(x, granularity, stream)
    sums = torch.empty(3, dtype=torch.float64, device=x.device)
    jf_quantization_error(x, q, s, GRANULARITY[granularity], sums, stream)
    if stream is not None:   # .item() below is ordered after the current stream only
        stream.synchronize() if hasattr(stream, "synchronize") else torch.cuda.synchronize()
    return float(sums[2].item())


def jf_mx_quantize(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_mx_quantize(_ptr(x), _DTYPES[x.dtype], x.shape[0], x.shape[1], _ptr(codes), _ptr(scales),
                              _stream(stream)), "jf_mx_quantize")


def jf_mx_linear_fwd(a_codes, a_scales, b_codes, b_scales, y: torch.Tensor, stream=None) -> None:
    lib = load_library()
    M, K = a_codes.shape
    N = b_codes.shape[0]
    _check(lib.jf_mx_linear_fwd(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K, _ptr(y),
                                _stream(stream)), "jf_mx_linear_fwd")


def mx_quantize(x: torch.Tensor, stream=None):
    """MXFP8 (E4M3 codes as uint8, E8M0 scale bytes per 1x32 block of a row) of x [rows, cols]."""
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((x.shape[0], x.shape[1] // 32), dtype=torch.uint8, device=x.device)
    jf_mx_quantize(x, codes, scales, stream)
    return codes, scales


def mx_linear_fwd(a_codes, a_scales, b_codes, b_scales, stream=None) -> torch.Tensor:
    """fp32 Y = A B^T of two MXFP8 tensors on the tensor core's block-scaled MMA."""
    y = torch.empty((a_codes.shape[0], b_codes.shape[0]), dtype=torch.float32, device=a_codes.device)
    jf_mx_linear_fwd(a_codes, a_scales, b_codes, b_scales, y, stream)
    return y


def jf_gemm_i8_s32(a: torch.Tensor, b: torch.Tensor, c: torch.Tensor, stream=None) -> None:
    """c (int32 [M, N]) = a (int8 [M, K]) @ b (int8 [N, K])^T on the tensor core, no scales."""
    lib = load_library()
    M, K = a.shape
    N = b.shape[0]
    _check(lib.jf_gemm_i8_s32(_ptr(a), _ptr(b), _ptr(c), M, N, K, _stream(stream)), "jf_gemm_i8_s32")


def jf_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    lib = load_library()
    _check(lib.jf_selftest_wait_timeout(limit_ns, _stream(stream)), "jf_selftest_wait_timeout")


def jf_strerror(status: int) -> str:
    return load_library().jf_strerror(int(status)).decode()


def jf_device_status(stream=None) -> int:
    return int(load_library().jf_device_status(_stream(stream)))


def jf_sm_count() -> int:
    return int(load_library().jf_sm_count())


# --------------------------------------------------------------------------- allocating helpers
def quantize_block(x: torch.Tensor, stream=None) -> QTensor:
    out = empty_qtensor(x.shape[0], x.shape[1], x.device)
    jf_quantize_block(x, out.q, out.s, stream)
    return out


def dequantize_block(t: QTensor, dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    y = torch.empty(t.q.shape, dtype=dtype, device=t.q.device)
    jf_dequantize_block(t.q, t.s, y, stream)
    return y


def linear_fwd(X: QTensor, W: QTensor, want_f32: bool = False, stream=None):
    Y = empty_qtensor(X.rows, W.rows, X.q.device)
    yf = torch.empty((X.rows, W.rows), dtype=torch.float32, device=X.q.device) if want_f32 else None
    jf_linear_fwd(X, W, Y, yf, stream)
    return (Y, yf) if want_f32 else Y


def linear_fwd_gelu(X: QTensor, W: QTensor, want_pre: bool = False, stream=None):
    """Y = requant(GELU(X W^T)) with GELU applied on chip; with ``want_pre`` also the re-quantized
    pre-activation (the same tensor linear_fwd returns)."""
    Y = empty_qtensor(X.rows, W.rows, X.q.device)
    P = empty_qtensor(X.rows, W.rows, X.q.device) if want_pre else None
    jf_linear_fwd_gelu(X, W, Y, P, stream)
    return (Y, P) if want_pre else Y


def linear_dgrad(dY: QTensor, W: QTensor, want_f32: bool = False, stream=None):
    dX = empty_qtensor(dY.rows, W.cols, dY.q.device)
    xf = torch.empty((dY.rows, W.cols), dtype=torch.float32, device=dY.q.device) if want_f32 else None
    jf_linear_dgrad(dY, W, dX, xf, stream)
    return (dX, xf) if want_f32 else dX


def linear_wgrad(dY: QTensor, X: QTensor, want_f32: bool = False, stream=None):
    dW = empty_qtensor(dY.cols, X.cols, dY.q.device)
    wf = torch.empty((dY.cols, X.cols), dtype=torch.float32, device=dY.q.device) if want_f32 else None
    jf_linear_wgrad(dY, X, dW, wf, stream)
    return (dW, wf) if want_f32 else dW


def gelu_i8(X: QTensor, stream=None) -> QTensor:
    Y = empty_qtensor(X.rows, X.cols, X.q.device)
    jf_gelu_i8(X, Y, stream)
    return Y


def gelu_i8_bwd(X: QTensor, dY: QTensor, stream=None) -> QTensor:
    """dX = requant(dY * GELU'(X)) on INT8 blocks; X is the saved pre-activation."""
    dX = empty_qtensor(X.rows, X.cols, X.q.device)
    jf_gelu_i8_bwd(X, dY, dX, stream)
    return dX


def layernorm_i8_bwd(X: QTensor, dY: QTensor, gamma: torch.Tensor, eps: float = 1e-5, stream=None):
    """(dX, dgamma, dbeta) of LayerNorm_i8; the workspace is allocated here, per call."""
    dX = empty_qtensor(X.rows, X.cols, X.q.device)
    dgamma = torch.empty(X.cols, dtype=torch.float32, device=X.q.device)
    dbeta = torch.empty_like(dgamma)
    ws = torch.empty(jf_layernorm_i8_bwd_workspace_bytes(X.rows, X.cols), dtype=torch.uint8, device=X.q.device)
    jf_layernorm_i8_bwd(X, dY, gamma, eps, dX, dgamma, dbeta, ws, stream)
    return dX, dgamma, dbeta


def layernorm_i8(X: QTensor, gamma: torch.Tensor, beta: torch.Tensor, eps: float = 1e-5, stream=None) -> QTensor:
    Y = empty_qtensor(X.rows, X.cols, X.q.device)
    jf_layernorm_i8(X, gamma, beta, eps, Y, stream)
    return Y



def quantize_block_rowstats(x: torch.Tensor, stream=None):
    """(QTensor, stats): the per-block quantization of x and, per row and block, the int32 sums of q
    and q^2 ([rows, cols/32, 2]) that layernorm_i8_rowstats takes in place of a pass over the codes."""
    out = empty_qtensor(x.shape[0], x.shape[1], x.device)
    stats = torch.empty((x.shape[0], x.shape[1] // 32, 2), dtype=torch.int32, device=x.device)
    jf_quantize_block_rowstats(x, out.q, out.s, stats, stream)
    return out, stats


def layernorm_i8_rowstats(X: QTensor, stats: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
                          eps: float = 1e-5, stream=None) -> QTensor:
    Y = empty_qtensor(X.rows, X.cols, X.q.device)
    jf_layernorm_i8_rowstats(X, stats, gamma, beta, eps, Y, stream)
    return Y